// tg_qkv_rope: the kept tokens' q/k/v projections with the rotary embedding at
// their original positions (MarkTechPost page on TokenGate, section "Comment
// TokenGate a-t-il appris le fonctionnement de la réduction des tokens ?": the
// layers above the gate layer process, and cache, only the K kept tokens).
//     y = W xc[r], W = [Wq; Wk; Wv];  q, k rotated at pos[r] (rotate-half pairs
//     (i, i + dh/2), theta_i = base^(-2i/dh));  v copied.
//
// One CTA per 256 rows x 256 output columns (two whole heads): a TMA producer
// thread streams, per stage, two 128x64 tiles of xc and one 256x64 tile of W
// (128-byte swizzle) through a 3-stage mbarrier ring; one thread issues, per K=16
// step, one tcgen05.mma (M=128, N=256, bf16 -> fp32) per row tile into its own
// 256-column TMEM accumulator (512 columns in all), both with the same W operand,
// so W is streamed once per 256 rows. Epilogue, all 16 warps, one row tile after
// the other: warp w reads TMEM lanes 32*(w%4).. and, of head (w/4)/2 of the tile,
// the pairs i in [32*((w/4)%2), +32) and i + 64, so every rotate-half pair is in
// one thread. The angle p*theta_i is formed in fp64 and reduced modulo 2 pi
// (positions reach 1e5 and more, where an fp32 product alone is off by ~1e-2 rad),
// then the fp32 sine and cosine of the reduced angle (MUFU, absolute error about
// 2^-21 on [-pi, pi]); the rotation and the bf16 rounding are fp32.
#include "common.cuh"

namespace {

constexpr int kBM = 128;      // rows per row tile (two row tiles per CTA)
constexpr int kBN = 256;      // output columns per tile: two heads of 128
constexpr int kBK = 64;
constexpr int kStages = 3;
constexpr int kThreads = 512;
constexpr int kDh = 128;
constexpr int kHalf = kDh / 2;

struct QkvSmem {
  uint8_t a[kStages][2][kBM * kBK * 2];   // two xc tiles, 16 KB each
  uint8_t b[kStages][kBN * kBK * 2];   // W tiles, 32 KB
  double theta[kHalf];                 // base^(-2i/dh)
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t acc_full;
  uint32_t tmem_base;
  int abort_flag;
};

__global__ void __launch_bounds__(kThreads, 1)
    qkv_rope_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                    int64_t n_rows, int d, int n_hq, int n_hkv, double log_base,
                    const int32_t* __restrict__ pos, __nv_bfloat16* __restrict__ q,
                    __nv_bfloat16* __restrict__ k, __nv_bfloat16* __restrict__ v, int* status) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (tg::smem_u32(smem_raw) & 1023u)) & 1023u;
  QkvSmem& S = *reinterpret_cast<QkvSmem*>(smem_raw + pad);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t m0 = static_cast<int64_t>(blockIdx.x) * (2 * kBM);
  const int n0 = blockIdx.y * kBN;   // first output column (= 128 * first head)
  const int nk = d / kBK;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      tg::mbar_init(&S.full[s], 1);
      tg::mbar_init(&S.empty[s], 1);
    }
    tg::mbar_init(&S.acc_full, 1);
    S.abort_flag = 0;
    tg::fence_barrier_init();
  }
  if (warp == 2) {
    tg::tmem_alloc(&S.tmem_base, 2 * kBN);
    tg::tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tg::tma_prefetch_desc(&tm_x);
    tg::tma_prefetch_desc(&tm_w);
  }
  if (tid >= 64 && tid < 64 + kHalf) {   // frequencies, fp64 (no global memory)
    const int i = tid - 64;
    S.theta[i] = exp(-2.0 * i / kDh * log_base);
  }
  tg::tc_fence_before();
  __syncthreads();
  tg::tc_fence_after();
  const uint32_t tmem = S.tmem_base;
  tg::pdl_launch_dependents();
  tg::pdl_wait();   // global memory only from here on

  if (warp == 0 && lane == 0) {
    // ---- TMA producer ----
    int issued = 0;
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % kStages;
      if (kb >= kStages &&
          !tg::mbar_wait(&S.empty[s], ((kb / kStages) - 1) & 1, status, &S.abort_flag))
        break;
      tg::mbar_arrive_expect_tx(&S.full[s], (2 * kBM + kBN) * kBK * 2);
      tg::tma_load_2d(S.a[s][0], &tm_x, &S.full[s], kb * kBK, static_cast<int>(m0));
      tg::tma_load_2d(S.a[s][1], &tm_x, &S.full[s], kb * kBK, static_cast<int>(m0 + kBM));
      tg::tma_load_2d(S.b[s], &tm_w, &S.full[s], kb * kBK, n0);
      ++issued;
    }
    if (S.abort_flag) {   // let copies already in flight land before the CTA can exit
      for (int kb = issued > kStages ? issued - kStages : 0; kb < issued; ++kb)
        tg::mbar_wait(&S.full[kb % kStages], (kb / kStages) & 1, status, nullptr);
    }
  } else if (warp == 1 && lane == 0) {
    // ---- MMA issuer ----
    constexpr uint32_t idesc = tg::idesc_bf16_f32(kBM, kBN, false, false);
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % kStages;
      if (!tg::mbar_wait(&S.full[s], (kb / kStages) & 1, status, &S.abort_flag)) break;
      tg::tc_fence_after();
      const uint32_t a0 = tg::smem_u32(S.a[s][0]), a1 = tg::smem_u32(S.a[s][1]);
      const uint32_t b0 = tg::smem_u32(S.b[s]);
#pragma unroll
      for (int kk = 0; kk < kBK / 16; ++kk) {
        const uint64_t bdesc = tg::smem_desc_sw128(b0 + 32 * kk, 16, 1024);
        const uint32_t acc = (kb > 0 || kk > 0) ? 1u : 0u;
        tg::mma_bf16_ss(tmem, tg::smem_desc_sw128(a0 + 32 * kk, 16, 1024), bdesc, idesc, acc);
        tg::mma_bf16_ss(tmem + kBN, tg::smem_desc_sw128(a1 + 32 * kk, 16, 1024), bdesc, idesc,
                        acc);
      }
      tg::mma_commit(&S.empty[s]);
    }
    tg::mma_commit(&S.acc_full);
  }
  __syncwarp();

  // ---- epilogue: all 16 warps, the two row tiles one after the other ----
  const int lg = warp & 3, cg = warp >> 2;
  const int hh = cg >> 1;                 // head within the tile
  const int i0 = (cg & 1) * 32;           // this thread's pairs: i0 .. i0+31 and +64
  const int gh = n0 / kDh + hh;           // global head index in [q heads, k heads, v heads]
  const bool ok = tg::mbar_wait(&S.acc_full, 0, status, &S.abort_flag);
  if (ok) tg::tc_fence_after();
#pragma unroll 1
  for (int rt = 0; rt < 2 && ok; ++rt) {
    const int64_t r = m0 + rt * kBM + lg * 32 + lane;   // row; TMEM lane lg*32 + lane
    uint32_t ya[32], yb[32];
    const uint32_t base =
        tmem + (static_cast<uint32_t>(lg * 32) << 16) + rt * kBN + hh * kDh + i0;
    tg::tmem_ld32(base, ya);
    tg::tmem_ld32(base + kHalf, yb);
    tg::tmem_ld_wait();
    if (r < n_rows) {
      __nv_bfloat16* dst;
      if (gh < n_hq) {
        dst = q + (r * n_hq + gh) * kDh;
      } else if (gh < n_hq + n_hkv) {
        dst = k + (r * n_hkv + (gh - n_hq)) * kDh;
      } else {
        dst = v + (r * n_hkv + (gh - n_hq - n_hkv)) * kDh;
      }
      uint32_t oa[16], ob[16];
      if (gh < n_hq + n_hkv) {   // q or k head: rotate each (i, i + 64) pair
        const double p = static_cast<double>(pos[r]);
        constexpr double kTwoPi = 6.283185307179586;
        constexpr double kInvTwoPi = 0.15915494309189535;
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float c[2], s[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const double ang = p * S.theta[i0 + e + u];
            const float red = static_cast<float>(fma(-kTwoPi, rint(ang * kInvTwoPi), ang));
            __sincosf(red, &s[u], &c[u]);   // |red| <= pi: absolute error ~2^-21
          }
          const float y1a = __uint_as_float(ya[e]), y1b = __uint_as_float(ya[e + 1]);
          const float y2a = __uint_as_float(yb[e]), y2b = __uint_as_float(yb[e + 1]);
          oa[e / 2] = tg::pack_bf16x2(y1a * c[0] - y2a * s[0], y1b * c[1] - y2b * s[1]);
          ob[e / 2] = tg::pack_bf16x2(y2a * c[0] + y1a * s[0], y2b * c[1] + y1b * s[1]);
        }
      } else {
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          oa[e / 2] = tg::pack_bf16x2(__uint_as_float(ya[e]), __uint_as_float(ya[e + 1]));
          ob[e / 2] = tg::pack_bf16x2(__uint_as_float(yb[e]), __uint_as_float(yb[e + 1]));
        }
      }
      uint4* da = reinterpret_cast<uint4*>(dst + i0);
      uint4* db = reinterpret_cast<uint4*>(dst + kHalf + i0);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        da[u] = make_uint4(oa[4 * u], oa[4 * u + 1], oa[4 * u + 2], oa[4 * u + 3]);
        db[u] = make_uint4(ob[4 * u], ob[4 * u + 1], ob[4 * u + 2], ob[4 * u + 3]);
      }
    }
  }
  tg::tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tg::tc_fence_after();
    tg::tmem_dealloc(tmem, 2 * kBN);
  }
}

}  // namespace

extern "C" tg_status tg_qkv_rope(const void* xc, int64_t n_rows, int d, const void* w_qkv,
                                 int n_hq, int n_hkv, int head_dim, float rope_base,
                                 const int32_t* pos, void* q, void* k, void* v,
                                 tg_stream_t stream) {
  tg::NvtxRange nvtx_range("tg_qkv_rope");
  if (n_rows < 0 || d <= 0 || n_hq <= 0 || n_hkv <= 0 || head_dim <= 0) return TG_ERR_INVALID_ARG;
  if (!(rope_base > 1.0f)) return TG_ERR_INVALID_ARG;
  if (n_rows == 0) return TG_OK;
  if (!xc || !w_qkv || !pos || !q || !k || !v) return TG_ERR_INVALID_ARG;
  if (head_dim != kDh || d % kBK != 0 || (n_hq + 2 * n_hkv) % 2 != 0) return TG_ERR_UNSUPPORTED;
  if (n_rows > INT32_MAX - kBM || (n_rows + kBM - 1) / kBM > INT32_MAX) return TG_ERR_UNSUPPORTED;
  const int64_t n_out = static_cast<int64_t>(n_hq + 2 * n_hkv) * kDh;
  if (n_out / kBN > 65535) return TG_ERR_UNSUPPORTED;
  if (!tg::aligned16(xc) || !tg::aligned16(w_qkv) || !tg::aligned16(q) || !tg::aligned16(k) ||
      !tg::aligned16(v))
    return TG_ERR_MISALIGNED;
  int* status = tg::status_word();
  if (!status) return TG_ERR_CUDA;
  CUtensorMap tx, tw;
  const uint64_t dx[2] = {static_cast<uint64_t>(d), static_cast<uint64_t>(n_rows)};
  const uint64_t sx[1] = {static_cast<uint64_t>(d) * 2};
  const uint32_t bx[2] = {kBK, kBM};
  const uint64_t dw[2] = {static_cast<uint64_t>(d), static_cast<uint64_t>(n_out)};
  const uint32_t bw[2] = {kBK, kBN};
  if (!tg::encode_tmap(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, xc, dx, sx, bx,
                       CU_TENSOR_MAP_SWIZZLE_128B) ||
      !tg::encode_tmap(&tw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w_qkv, dw, sx, bw,
                       CU_TENSOR_MAP_SWIZZLE_128B))
    return TG_ERR_CUDA;
  const size_t smem = sizeof(QkvSmem) + 1024;
  if (!tg::ensure_smem(reinterpret_cast<const void*>(qkv_rope_kernel), static_cast<int>(smem)))
    return TG_ERR_CUDA;
  const dim3 grid(static_cast<unsigned>((n_rows + 2 * kBM - 1) / (2 * kBM)),
                  static_cast<unsigned>(n_out / kBN));
  return tg::launch(qkv_rope_kernel, grid, dim3(kThreads), smem, stream, 0, tx, tw, n_rows, d, n_hq,
                    n_hkv, log(static_cast<double>(rope_base)), pos,
                    static_cast<__nv_bfloat16*>(q), static_cast<__nv_bfloat16*>(k),
                    static_cast<__nv_bfloat16*>(v), status);
}

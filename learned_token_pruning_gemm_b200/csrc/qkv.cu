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
// so W is streamed once per 256 rows. The rotary angles do not depend on the
// products, so the warps that wait on the accumulators take them while the MMAs
// run: the angle of position p and frequency i, in turns, is p * F_i mod 1 with
// F_i = theta_i / (2 pi) held as a 64-bit fixed-point fraction (one integer
// product, exact modulo 2^64; positions reach 1e5 and more, where an fp32 product
// alone is off by ~1e-2 rad), rounded to 23 bits and brought to [-pi, pi) in
// fp32, then the fp32 sine and cosine (MUFU, absolute error about 2^-21). The two
// heads of a tile share their rows' angles: each of a pair of warps takes half of
// them and hands its half over through the freed stage buffers. Epilogue, all 16
// warps, one row tile after the other: warp w reads TMEM lanes 32*(w%4).. and, of
// head (w/4)/2 of the tile, the pairs i in [32*((w/4)%2), +32) and i + 64, so
// every rotate-half pair is in one thread; the rotation and the bf16 rounding are
// fp32; the rows are staged in shared memory as the output maps' boxes (64 columns
// x 128 rows, 128-byte swizzle) and leave as TMA tensor stores, so the second row
// tile's rotation runs while the first one's stores drain (rows past the last are
// clipped by the maps).
//
// tg_compact_qkv_rope runs the same kernel on the rows of the full residual named
// by kept_idx, so the compaction is fused into the projection: four warps that
// otherwise only wait on the accumulators gather each stage's 2 x 128 rows x 128
// bytes with 16-byte cp.async copies straight into the swizzled stage layout
// (each thread one 16-byte column of 16 rows; rows past the end are zero-filled),
// and the stage completes on their arrivals plus the W tile's TMA bytes; the MMA
// thread orders those generic-proxy writes before its tensor-core reads with a
// proxy fence. The compacted rows are written out on the way: of every k-block,
// the CTAs of one column tile load it through registers and store it to xc too.
#include "common.cuh"

namespace {

constexpr int kBM = 128;      // rows per row tile (two row tiles per CTA)
constexpr int kBN = 256;      // output columns per tile: two heads of 128
constexpr int kBK = 64;
constexpr int kStages = 3;
constexpr int kThreads = 512;
constexpr int kDh = 128;
constexpr int kHalf = kDh / 2;

constexpr int kGatherWarp0 = 12;             // gather mode: warps 12..15 gather the rows
constexpr int kGatherThreads = kThreads - kGatherWarp0 * 32;
static_assert(kGatherThreads == 128, "one 16-byte column of 16 rows per gather thread");

// 16 bytes global -> shared, or 16 zero bytes when !ok (src is not read then)
__device__ __forceinline__ void cp16(void* dst, const void* src, bool ok) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(tg::smem_u32(dst)), "l"(src),
               "r"(ok ? 16 : 0)
               : "memory");
}
// one arrival on bar once this thread's earlier cp.async copies have landed
__device__ __forceinline__ void cp_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(tg::smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void cp_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

struct QkvSmem {
  uint8_t a[kStages][2][kBM * kBK * 2];   // two xc tiles, 16 KB each
  uint8_t b[kStages][kBN * kBK * 2];   // W tiles, 32 KB
  uint64_t turn[kHalf];                // theta_i / (2 pi) in 0.64 fixed point
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t acc_full;
  uint32_t tmem_base;
  int abort_flag;
};

// kGather: the rows are x[kept_idx[r]] (n_src rows of x), gathered by warps 12..15,
// and xc (if not null) receives them; otherwise tm_x maps the compacted rows.
template <bool kGather>
__global__ void __launch_bounds__(kThreads, 1)
    qkv_rope_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                    const __grid_constant__ CUtensorMap tm_oq, const __grid_constant__ CUtensorMap tm_ok,
                    const __grid_constant__ CUtensorMap tm_ov,
                    int64_t n_rows, int d, int n_hq, int n_hkv, double log_base,
                    const int32_t* __restrict__ pos, __nv_bfloat16* __restrict__ q,
                    __nv_bfloat16* __restrict__ k, __nv_bfloat16* __restrict__ v,
                    const __nv_bfloat16* __restrict__ x, int64_t n_src,
                    const int32_t* __restrict__ kept_idx, __nv_bfloat16* __restrict__ xc,
                    int* status) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (tg::smem_u32(smem_raw) & 1023u)) & 1023u;
  QkvSmem& S = *reinterpret_cast<QkvSmem*>(smem_raw + pad);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t m0 = static_cast<int64_t>(blockIdx.x) * (2 * kBM);
  const int n0 = blockIdx.y * kBN;   // first output column (= 128 * first head)
  const int nk = d / kBK;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      tg::mbar_init(&S.full[s], kGather ? 1 + kGatherThreads : 1);
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
    if (!kGather) tg::tma_prefetch_desc(&tm_x);
    tg::tma_prefetch_desc(&tm_w);
  }
  if (tid >= 64 && tid < 64 + kHalf) {   // frequencies (no global memory)
    const int i = tid - 64;
    constexpr double kInvTwoPi = 0.15915494309189535;
    S.turn[i] = __double2ull_rn(ldexp(exp(-2.0 * i / kDh * log_base) * kInvTwoPi, 64));
  }
  tg::tc_fence_before();
  __syncthreads();
  tg::tc_fence_after();
  const uint32_t tmem = S.tmem_base;
  tg::pdl_launch_dependents();
  tg::pdl_wait();   // global memory only from here on

  const int lg = warp & 3, cg = warp >> 2;
  const int hh = cg >> 1;                 // head within the tile
  const int i0 = (cg & 1) * 32;           // this thread's pairs: i0 .. i0+31 and +64
  const int gh0 = n0 / kDh;               // global head index of head 0 of the tile
  const bool rope = gh0 < n_hq + n_hkv;   // head 0 (and so any head before v) is rotated
  const int row = lg * 32 + lane;         // row within a row tile; TMEM lane
  // this thread's half of its rows' angles: i in [i0 + 16 hh, +16), both row tiles;
  // (c, s) = (-cos, -sin) of the angle less pi, i.e. cos and sin of the angle itself
  float2 cs[2][16];
  auto angles = [&]() {
#pragma unroll
    for (int rt = 0; rt < 2; ++rt) {
      const int64_t r = m0 + rt * kBM + row;
      const int p = r < n_rows ? pos[r] : 0;
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const uint64_t fx = static_cast<uint64_t>(static_cast<int64_t>(p)) * S.turn[i0 + 16 * hh + e];
        const uint32_t fr = static_cast<uint32_t>(fx >> 32);   // turns mod 1, top 32 bits
        // to 23 bits as a float in [1, 2] (a carry out of the top wraps to 1 turn == 0)
        const float f1 = __uint_as_float(0x3F800000u + ((fr + 256u) >> 9));
        const float x = (f1 - 1.5f) * 6.28318530717958648f;   // 2 pi (turns - 1/2), |x| <= pi
        float sn, cn;
        __sincosf(x, &sn, &cn);   // |x| <= pi: absolute error ~2^-21
        cs[rt][e] = make_float2(-cn, -sn);
      }
    }
  };
  const bool gather_warp = kGather && warp >= kGatherWarp0;
  if (rope && warp >= 2 && !gather_warp) angles();   // under the mainloop: these warps only wait


  if (warp == 0 && lane == 0) {
    // ---- TMA producer ----
    int issued = 0;
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % kStages;
      if (kb >= kStages &&
          !tg::mbar_wait(&S.empty[s], ((kb / kStages) - 1) & 1, status, &S.abort_flag))
        break;
      if (kGather) {   // W only: the rows come from the gather warps
        tg::mbar_arrive_expect_tx(&S.full[s], kBN * kBK * 2);
      } else {
        tg::mbar_arrive_expect_tx(&S.full[s], (2 * kBM + kBN) * kBK * 2);
        tg::tma_load_2d(S.a[s][0], &tm_x, &S.full[s], kb * kBK, static_cast<int>(m0));
        tg::tma_load_2d(S.a[s][1], &tm_x, &S.full[s], kb * kBK, static_cast<int>(m0 + kBM));
      }
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
      if (kGather) tg::fence_proxy_async_shared();   // the gathered rows: generic-proxy writes
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
  } else if (gather_warp) {
    // ---- row gather: thread gt owns 16-byte column c of rows r0 + 16u, u < 16, of
    //      the stage's two row tiles (a warp covers four whole 128-byte rows) ----
    const int gt = tid - kGatherWarp0 * 32;
    const int c = gt & 7, r0 = gt >> 3;
    int32_t src[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) {
      const int64_t r = m0 + r0 + 16 * u;
      int32_t sr = -1;
      if (r < n_rows) {
        sr = kept_idx[r];
        if (sr < 0 || sr >= n_src) {   // not a row of x: zeros, and the error recorded
          tg::set_status(status, TG_ERR_DEVICE_CHECK);
          sr = -1;
        }
      }
      src[u] = sr;
    }
    const int n_ct = static_cast<int>(gridDim.y);
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % kStages;
      if (kb >= kStages &&
          !tg::mbar_wait(&S.empty[s], ((kb / kStages) - 1) & 1, status, &S.abort_flag))
        break;
      const int64_t col = static_cast<int64_t>(kb) * kBK + 8 * c;
      if (xc && kb % n_ct == static_cast<int>(blockIdx.y)) {
        // this CTA also writes k-block kb of the compacted rows: through registers
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const int r = r0 + 16 * u, rr = r & (kBM - 1);
          uint4 val = make_uint4(0, 0, 0, 0);
          if (src[u] >= 0) {
            val = *reinterpret_cast<const uint4*>(x + static_cast<int64_t>(src[u]) * d + col);
            if (tg::in_bounds(m0 + r, n_rows, status))
              *reinterpret_cast<uint4*>(xc + (m0 + r) * d + col) = val;
          }
          *reinterpret_cast<uint4*>(S.a[s][r >> 7] + rr * 128 + ((c ^ (rr & 7)) << 4)) = val;
        }
        tg::mbar_arrive(&S.full[s]);
      } else {
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const int r = r0 + 16 * u, rr = r & (kBM - 1);
          const bool ok = src[u] >= 0;
          cp16(S.a[s][r >> 7] + rr * 128 + ((c ^ (rr & 7)) << 4),
               x + (ok ? static_cast<int64_t>(src[u]) * d + col : 0), ok);
        }
        cp_arrive(&S.full[s]);
      }
    }
    cp_wait_all();   // no copy may land after the CTA has moved on
  }
  __syncwarp();
  if (rope && (warp < 2 || gather_warp)) angles();

  // ---- epilogue: all 16 warps ----
  // Once the accumulators are complete every stage has been consumed, so the stage
  // buffers (192 KB) hold: the angle tables of the two row tiles, [i][row] float2
  // (64 KB each), and the bf16 output rows of one row tile (64 KB).
  const bool ok = tg::mbar_wait(&S.acc_full, 0, status, &S.abort_flag);
  if (ok) tg::tc_fence_after();
  uint8_t* const base = &S.a[0][0][0];
  float2* const table = reinterpret_cast<float2*>(base);   // [rt][i][row]
  if (rope && ok) {
#pragma unroll
    for (int rt = 0; rt < 2; ++rt)
#pragma unroll
      for (int e = 0; e < 16; ++e) table[(rt * kHalf + i0 + 16 * hh + e) * kBM + row] = cs[rt][e];
  }
  const bool rot = gh0 + hh < n_hq + n_hkv;   // this thread's head is q or k
  __syncthreads();   // angle tables written
#pragma unroll 1
  for (int rt = 0; rt < 2; ++rt) {
    // output staging, four 16 KB boxes (head h, 64-column half j) of 128 rows x 128 B,
    // 16-byte pieces swizzled as the output maps' 128-byte swizzle expects: row tile 0
    // after the tables, row tile 1 over table 0 (read by then)
    uint8_t* const stg = rt == 0 ? base + 2 * kHalf * kBM * sizeof(float2) : base;
    if (ok) {
      uint32_t ya[32], yb[32];
      const uint32_t taddr =
          tmem + (static_cast<uint32_t>(lg * 32) << 16) + rt * kBN + hh * kDh + i0;
      tg::tmem_ld32(taddr, ya);
      tg::tmem_ld32(taddr + kHalf, yb);
      tg::tmem_ld_wait();
      uint32_t oa[16], ob[16];
      if (rot) {   // rotate each (i, i + 64) pair
        const float2* tb = table + (rt * kHalf + i0) * kBM + row;
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const float2 c0 = tb[e * kBM], c1 = tb[(e + 1) * kBM];
          const float y1a = __uint_as_float(ya[e]), y1b = __uint_as_float(ya[e + 1]);
          const float y2a = __uint_as_float(yb[e]), y2b = __uint_as_float(yb[e + 1]);
          oa[e / 2] = tg::pack_bf16x2(y1a * c0.x - y2a * c0.y, y1b * c1.x - y2b * c1.y);
          ob[e / 2] = tg::pack_bf16x2(y2a * c0.x + y1a * c0.y, y2b * c1.x + y1b * c1.y);
        }
      } else {
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          oa[e / 2] = tg::pack_bf16x2(__uint_as_float(ya[e]), __uint_as_float(ya[e + 1]));
          ob[e / 2] = tg::pack_bf16x2(__uint_as_float(yb[e]), __uint_as_float(yb[e + 1]));
        }
      }
      // oa: columns i0.. of half 0, ob: the same of half 1; piece i0/8 + u of the row
      uint8_t* const ra = stg + (hh * 2) * (kBM * 128) + row * 128;
      uint8_t* const rb = ra + kBM * 128;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int off = (((i0 >> 3) + u) ^ (row & 7)) << 4;
        *reinterpret_cast<uint4*>(ra + off) =
            make_uint4(oa[4 * u], oa[4 * u + 1], oa[4 * u + 2], oa[4 * u + 3]);
        *reinterpret_cast<uint4*>(rb + off) =
            make_uint4(ob[4 * u], ob[4 * u + 1], ob[4 * u + 2], ob[4 * u + 3]);
      }
    }
    tg::fence_proxy_async_shared();   // the staged rows, to the TMA unit
    __syncthreads();
    if (ok && tid == 0) {
      // four boxes out; rows past the last are clipped by the maps' extent
      const int z = static_cast<int>(m0 + rt * kBM);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int gh = gh0 + h;
        const CUtensorMap* m = gh < n_hq ? &tm_oq : gh < n_hq + n_hkv ? &tm_ok : &tm_ov;
        const int y = gh < n_hq ? gh : gh < n_hq + n_hkv ? gh - n_hq : gh - n_hq - n_hkv;
#pragma unroll
        for (int j = 0; j < 2; ++j)
          tg::tma_store_3d(m, stg + (h * 2 + j) * (kBM * 128), 64 * j, y, z);
      }
      tg::bulk_commit();
    }
  }
  if (tid == 0) tg::bulk_wait_read_all();   // the boxes stay in place until read
  tg::tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tg::tc_fence_after();
    tg::tmem_dealloc(tmem, 2 * kBN);
  }
}

}  // namespace

namespace {

// both entry points: validation, the W map (and the xc map unless gathering), launch
tg_status launch_qkv(const void* xc, const void* x, int64_t n_src, const int32_t* kept_idx,
                     void* xc_out, int64_t n_rows, int d, const void* w_qkv, int n_hq, int n_hkv,
                     int head_dim, float rope_base, const int32_t* pos, void* q, void* k, void* v,
                     cudaStream_t stream) {
  const bool gather = x != nullptr;
  if (n_rows < 0 || d <= 0 || n_hq <= 0 || n_hkv <= 0 || head_dim <= 0) return TG_ERR_INVALID_ARG;
  if (gather && n_src <= 0) return TG_ERR_INVALID_ARG;
  if (!(rope_base > 1.0f)) return TG_ERR_INVALID_ARG;
  if (n_rows == 0) return TG_OK;
  if ((gather ? !kept_idx : !xc) || !w_qkv || !pos || !q || !k || !v) return TG_ERR_INVALID_ARG;
  if (head_dim != kDh || d % kBK != 0 || (n_hq + 2 * n_hkv) % 2 != 0) return TG_ERR_UNSUPPORTED;
  if (n_rows > INT32_MAX - kBM || (n_rows + kBM - 1) / kBM > INT32_MAX) return TG_ERR_UNSUPPORTED;
  if (gather && n_src > INT32_MAX) return TG_ERR_UNSUPPORTED;
  const int64_t n_out = static_cast<int64_t>(n_hq + 2 * n_hkv) * kDh;
  if (n_out / kBN > 65535) return TG_ERR_UNSUPPORTED;
  if (!tg::aligned16(gather ? x : xc) || !tg::aligned16(w_qkv) || !tg::aligned16(q) ||
      !tg::aligned16(k) || !tg::aligned16(v) || (xc_out && !tg::aligned16(xc_out)))
    return TG_ERR_MISALIGNED;
  int* status = tg::status_word();
  if (!status) return TG_ERR_CUDA;
  CUtensorMap tx = {}, tw;
  const uint64_t sx[1] = {static_cast<uint64_t>(d) * 2};
  const uint64_t dw[2] = {static_cast<uint64_t>(d), static_cast<uint64_t>(n_out)};
  const uint32_t bw[2] = {kBK, kBN};
  if (!tg::encode_tmap(&tw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w_qkv, dw, sx, bw,
                       CU_TENSOR_MAP_SWIZZLE_128B))
    return TG_ERR_CUDA;
  if (!gather) {
    const uint64_t dx[2] = {static_cast<uint64_t>(d), static_cast<uint64_t>(n_rows)};
    const uint32_t bx[2] = {kBK, kBM};
    if (!tg::encode_tmap(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, xc, dx, sx, bx,
                         CU_TENSOR_MAP_SWIZZLE_128B))
      return TG_ERR_CUDA;
  }
  // the outputs, [n_rows, heads, 128] each, stored as 64-column x 128-row boxes
  CUtensorMap toq, tok, tov;
  const uint32_t bo[3] = {64, 1, kBM};
  const uint64_t oq_d[3] = {kDh, static_cast<uint64_t>(n_hq), static_cast<uint64_t>(n_rows)};
  const uint64_t oq_s[2] = {kDh * 2, static_cast<uint64_t>(n_hq) * kDh * 2};
  const uint64_t ok_d[3] = {kDh, static_cast<uint64_t>(n_hkv), static_cast<uint64_t>(n_rows)};
  const uint64_t ok_s[2] = {kDh * 2, static_cast<uint64_t>(n_hkv) * kDh * 2};
  if (!tg::encode_tmap(&toq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, q, oq_d, oq_s, bo,
                       CU_TENSOR_MAP_SWIZZLE_128B) ||
      !tg::encode_tmap(&tok, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, k, ok_d, ok_s, bo,
                       CU_TENSOR_MAP_SWIZZLE_128B) ||
      !tg::encode_tmap(&tov, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, v, ok_d, ok_s, bo,
                       CU_TENSOR_MAP_SWIZZLE_128B))
    return TG_ERR_CUDA;
  const size_t smem = sizeof(QkvSmem) + 1024;
  auto kernel = gather ? qkv_rope_kernel<true> : qkv_rope_kernel<false>;
  if (!tg::ensure_smem(reinterpret_cast<const void*>(kernel), static_cast<int>(smem)))
    return TG_ERR_CUDA;
  const dim3 grid(static_cast<unsigned>((n_rows + 2 * kBM - 1) / (2 * kBM)),
                  static_cast<unsigned>(n_out / kBN));
  return tg::launch(kernel, grid, dim3(kThreads), smem, stream, 0, tx, tw, toq, tok, tov, n_rows, d,
                    n_hq, n_hkv,
                    log(static_cast<double>(rope_base)), pos, static_cast<__nv_bfloat16*>(q),
                    static_cast<__nv_bfloat16*>(k), static_cast<__nv_bfloat16*>(v),
                    static_cast<const __nv_bfloat16*>(x), n_src, kept_idx,
                    static_cast<__nv_bfloat16*>(xc_out), status);
}

}  // namespace

extern "C" tg_status tg_qkv_rope(const void* xc, int64_t n_rows, int d, const void* w_qkv,
                                 int n_hq, int n_hkv, int head_dim, float rope_base,
                                 const int32_t* pos, void* q, void* k, void* v,
                                 tg_stream_t stream) {
  tg::NvtxRange nvtx_range("tg_qkv_rope");
  if (!xc && n_rows > 0) return TG_ERR_INVALID_ARG;
  return launch_qkv(xc, nullptr, 0, nullptr, nullptr, n_rows, d, w_qkv, n_hq, n_hkv, head_dim,
                    rope_base, pos, q, k, v, stream);
}

extern "C" tg_status tg_compact_qkv_rope(const void* x, int64_t n_src, int d,
                                         const int32_t* kept_idx, int64_t n_rows, void* xc,
                                         const void* w_qkv, int n_hq, int n_hkv, int head_dim,
                                         float rope_base, const int32_t* pos, void* q, void* k,
                                         void* v, tg_stream_t stream) {
  tg::NvtxRange nvtx_range("tg_compact_qkv_rope");
  if (!x && n_rows > 0) return TG_ERR_INVALID_ARG;
  return launch_qkv(nullptr, x, n_src, kept_idx, xc, n_rows, d, w_qkv, n_hq, n_hkv, head_dim,
                    rope_base, pos, q, k, v, stream);
}

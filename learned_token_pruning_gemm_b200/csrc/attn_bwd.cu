// tg_gated_attention_bwd: gradients of the token-gated attention (MarkTechPost page
// on TokenGate, section "Qu'est-ce que l'attention gérée par des tokens ?": the key
// score enters the logits as a bias precisely so that gradients reach the scorer;
// the per-head gain and temperature are learned).
//   z_ij = c_h q_i.k_j + g_h s_j (c_h = 1/(sqrt(dh) tau_h)),  P = softmax_j(z),
//   dP_ij = dO_i.v_j,  D_i = dO_i.O_i,  dZ_ij = P_ij (dP_ij - D_i)
//   dq_i = c_h sum_j dZ_ij k_j      dk_j = sum_h c_h sum_i dZ_ij q_i
//   dv_j = sum_h sum_i P_ij dO_i    ds_j = sum_h g_h sum_i dZ_ij
//   dg_h = sum_ij dZ_ij s_j         dtau_h = -(c_h / tau_h) sum_ij dZ_ij (q_i.k_j)
// P is rebuilt from the forward's log-sum-exp of each row, so no row reduction is
// needed here: every step is elementwise or a contraction.
//
// bf16 path (dh = 128), four kernels:
//   prep        D_i = dO_i.O_i and the log-sum-exp in log2 units, [n_hq, total] f32
//               in the workspace.
//   dq          one CTA per (query tile, query head): for each key tile j,
//               S = Q K_j^T and dP = dO V_j^T (tcgen05, TMEM), the elementwise
//               warps form dS = c_h P (dP - D) in bf16 over S, and dQ += dS K_j
//               (A from TMEM, K_j as an MN-major operand) accumulates in TMEM.
//   dkdv        one CTA per (key tile, KV head): for every query head of the group
//               and every query tile at or after the key tile, S^T = K Q^T and
//               dP^T = V dO^T (keys on the TMEM lanes); P^T and c_h dS^T go back
//               over them in bf16; dV += P^T dO and dK += dS^T Q accumulate in TMEM
//               over all of them, so each dK/dV row is written once, by one CTA,
//               with no atomics. The same threads sum each key's dZ row (score
//               gradient) and the CTA's dZ.s and dZ.qk (gain and temperature).
//   reduce      ds_j over KV heads, dg_h and dtau_h over CTAs, in a fixed order.
// f32 path (exact SIMT, small problems): the same prep and reduce, with one warp
// per (row, head) for dq and one warp per (key, KV head) for dk, dv.
#include "common.cuh"

namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kD = 128;
constexpr int kBM = 128;   // query rows per tile
constexpr int kBN = 128;   // keys per tile
constexpr int kBwdThreads = 256;   // warps 0-3 elementwise, 4 TMA, 5 MMA, 6 loader, 7 TMEM

__device__ __forceinline__ uint32_t tmem_lane_addr(uint32_t base, int warp, uint32_t col) {
  return base + (static_cast<uint32_t>(warp * 32) << 16) + col;
}

// ------------------------------------------------------------------------- //
// workspace layout (bytes, all f32)                                          //
// ------------------------------------------------------------------------- //
struct BwdWs {
  float* D;      // [n_hq, total]
  float* lse2;   // [n_hq, total]   log-sum-exp in log2 units
  float* ds;     // partial score gradients: bf16 [2 halves, n_hkv, total], f32 [n_hkv, total]
  float* gt;     // gain / temperature partials: bf16 [n_cta, group, 4 warps, 2],
                 // f32 [total, n_hq, 1, 2]
  float* dkv;    // bf16: dK and dV partials [2 halves][2 (dk, dv)][total, n_hkv, dh] fp32
};
// With at most kSplitMaxUnits (key tile, KV head, sequence) units the grid is one
// wave and the longest units set the time: each is then split between kKvSplit CTAs
// (halves of its items) that write fp32 partials, summed by the reduction. With more
// units they run whole and write dK and dV directly.
constexpr int kKvSplit = 2;
constexpr int kSplitMaxUnits = 128;
inline int kv_split(int64_t units) { return units <= kSplitMaxUnits ? kKvSplit : 1; }

// D_i = dO_i . O_i and lse2 = lse * log2(e); one warp per (row, head)
template <typename T>
__global__ void __launch_bounds__(256)
    bwd_prep_kernel(const T* __restrict__ out, const T* __restrict__ dout,
                    const float* __restrict__ lse, int64_t total, int n_hq, int dh,
                    float* __restrict__ D, float* __restrict__ lse2) {
  tg::pdl_launch_dependents();
  tg::pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t w = (static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x) >> 5;
  if (w >= total * n_hq) return;
  const int64_t row = w / n_hq;
  const int h = static_cast<int>(w % n_hq);
  const T* o = out + w * dh;
  const T* d = dout + w * dh;
  float acc = 0.f;
  for (int e = lane; e < dh; e += 32) {
    float oe, de;
    if constexpr (sizeof(T) == 2) {
      oe = __bfloat162float(o[e]);
      de = __bfloat162float(d[e]);
    } else {
      oe = o[e];
      de = d[e];
    }
    acc = fmaf(oe, de, acc);
  }
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, off);
  if (lane == 0) {
    D[static_cast<int64_t>(h) * total + row] = acc;
    lse2[static_cast<int64_t>(h) * total + row] = lse[static_cast<int64_t>(h) * total + row] * kLog2e;
  }
}

// ------------------------------------------------------------------------- //
// bf16: dQ                                                                   //
// ------------------------------------------------------------------------- //
struct DqSmem {
  uint8_t q[2][kBM * 64 * 2];          // Q_i, two 64-dim halves
  uint8_t dout[2][kBM * 64 * 2];       // dO_i
  uint8_t k[2][2][kBN * 64 * 2];       // K_j ring
  uint8_t v[2][2][kBN * 64 * 2];       // V_j ring
  float bias[2][kBN];                  // log2(e) g_h s_j of the ring's key tiles
  uint64_t qd_full;
  uint64_t kv_full[2], kv_empty[2];
  uint64_t b_full[2], b_empty[2];
  uint64_t sp_full[2], ds_full[2], dq_done;   // per 64-key half of the key tile
  uint32_t tmem_base;
  int abort_flag;
};
constexpr uint32_t kColS = 0, kColDP = 128, kColAcc = 256;

__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                  const float* __restrict__ s_kept, const float* __restrict__ gain,
                  const float* __restrict__ tau, const int32_t* __restrict__ cu_kept, int total,
                  int max_kept, int n_hq, int n_hkv, const float* __restrict__ D,
                  const float* __restrict__ lse2, __nv_bfloat16* __restrict__ dq, int* status) {
  const int hq = blockIdx.x;
  const int t = static_cast<int>(gridDim.y) - 1 - static_cast<int>(blockIdx.y);   // longest first
  const int b = blockIdx.z;
  const int kvh = hq / (n_hq / n_hkv);
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (tg::smem_u32(smem_raw) & 1023u)) & 1023u;
  DqSmem& S = *reinterpret_cast<DqSmem*>(smem_raw + pad);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    tg::mbar_init(&S.qd_full, 1);
    for (int i = 0; i < 2; ++i) {
      tg::mbar_init(&S.kv_full[i], 1);
      tg::mbar_init(&S.kv_empty[i], 1);
      tg::mbar_init(&S.b_full[i], 32);
      tg::mbar_init(&S.b_empty[i], 4);
    }
    for (int i = 0; i < 2; ++i) {
      tg::mbar_init(&S.sp_full[i], 1);
      tg::mbar_init(&S.ds_full[i], 4);
    }
    tg::mbar_init(&S.dq_done, 1);
    S.abort_flag = 0;
    tg::fence_barrier_init();
  }
  if (warp == 7) {
    tg::tmem_alloc(&S.tmem_base, 512);
    tg::tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    tg::tma_prefetch_desc(&tm_q);
    tg::tma_prefetch_desc(&tm_k);
    tg::tma_prefetch_desc(&tm_v);
    tg::tma_prefetch_desc(&tm_do);
  }
  tg::tc_fence_before();
  __syncthreads();
  tg::tc_fence_after();
  const uint32_t tmem = S.tmem_base;
  tg::pdl_launch_dependents();
  tg::pdl_wait();

  const int seq0 = cu_kept[b], seq1 = cu_kept[b + 1];
  const bool bad = seq0 < 0 || seq1 < seq0 || seq1 > total || seq1 - seq0 > max_kept;
  if (bad && hq == 0 && t == static_cast<int>(gridDim.y) - 1 && tid == 0)
    tg::set_status(status, TG_ERR_DEVICE_CHECK);
  const int len = bad ? 0 : seq1 - seq0;
  if (t * kBM >= len) {
    if (warp == 7) tg::tmem_dealloc(tmem, 512);
    return;
  }
  const int nt = t + 1;   // key tiles 0..t

  if (warp == 4) {
    // ---- TMA: Q and dO once, then the K/V ring ----
    if (lane == 0) {
      tg::mbar_arrive_expect_tx(&S.qd_full, 2 * kBM * kD * 2);
      for (int hh = 0; hh < 2; ++hh) {
        tg::tma_load_3d(S.q[hh], &tm_q, &S.qd_full, 64 * hh, hq, seq0 + t * kBM);
        tg::tma_load_3d(S.dout[hh], &tm_do, &S.qd_full, 64 * hh, hq, seq0 + t * kBM);
      }
      int j = 0;
      for (; j < nt; ++j) {
        const int st = j & 1;
        if (j >= 2 && !tg::mbar_wait(&S.kv_empty[st], ((j >> 1) - 1) & 1, status, &S.abort_flag)) break;
        tg::mbar_arrive_expect_tx(&S.kv_full[st], 2 * kBN * kD * 2);
        for (int hh = 0; hh < 2; ++hh) {
          tg::tma_load_3d(S.k[st][hh], &tm_k, &S.kv_full[st], 64 * hh, kvh, seq0 + j * kBN);
          tg::tma_load_3d(S.v[st][hh], &tm_v, &S.kv_full[st], 64 * hh, kvh, seq0 + j * kBN);
        }
      }
      if (S.abort_flag) {
        tg::mbar_wait(&S.qd_full, 0, status, nullptr);
        for (int i = j > 2 ? j - 2 : 0; i < j; ++i)
          tg::mbar_wait(&S.kv_full[i & 1], (i >> 1) & 1, status, nullptr);
      }
    }
    __syncwarp();
  } else if (warp == 5) {
    // ---- MMA: S = Q K^T, dP = dO V^T, then dQ += dS K, by 64-key halves ----
    // Order S_lo dP_lo, S_hi dP_hi, dQ_lo, [next tile] S_lo dP_lo, dQ_hi, S_hi dP_hi,
    // dQ_lo, ...: the elementwise warps work on one half while the tensor core
    // computes the other. A half's S and dP are rewritten only after the dQ MMA that
    // reads its dS was issued (the pipe runs in order) and its dP was read.
    if (lane == 0) {
      constexpr uint32_t idesc_h = tg::idesc_bf16_f32(kBM, kBN / 2, false, false);
      constexpr uint32_t idesc_q = tg::idesc_bf16_f32(kBM, kD, false, true);
      bool alive = tg::mbar_wait(&S.qd_full, 0, status, &S.abort_flag);
      const uint32_t q0 = tg::smem_u32(S.q[0]), d0 = tg::smem_u32(S.dout[0]);
      // S and dP of half h of key tile j (keys 64h .. 64h+63: rows 64h of the
      // 128-byte-swizzled K and V tiles, 8 KB into each 64-dim half)
      auto issue_sp = [&](int j, int h) -> bool {
        const int st = j & 1;
        if (h == 0 && !tg::mbar_wait(&S.kv_full[st], (j >> 1) & 1, status, &S.abort_flag))
          return false;
        tg::tc_fence_after();
        const uint32_t k0 = tg::smem_u32(S.k[st][0]) + h * (kBN / 2) * 128;
        const uint32_t v0 = tg::smem_u32(S.v[st][0]) + h * (kBN / 2) * 128;
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (kBM * 64 * 2) + (kk & 3) * 32;
          tg::mma_bf16_ss(tmem + kColS + 64 * h, tg::smem_desc_sw128(q0 + off, 16, 1024),
                          tg::smem_desc_sw128(k0 + off, 16, 1024), idesc_h, kk != 0);
        }
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (kBM * 64 * 2) + (kk & 3) * 32;
          tg::mma_bf16_ss(tmem + kColDP + 64 * h, tg::smem_desc_sw128(d0 + off, 16, 1024),
                          tg::smem_desc_sw128(v0 + off, 16, 1024), idesc_h, kk != 0);
        }
        tg::mma_commit(&S.sp_full[h]);
        return true;
      };
      // dQ += dS_h K_h: A = dS of half h (packed bf16 at columns 64h .. 64h+31 of S,
      // 8 columns per 16 keys), B = K rows 64h + 16kk .. as an MN-major operand
      auto issue_dq = [&](int j, int h) -> bool {
        if (!tg::mbar_wait(&S.ds_full[h], j & 1, status, &S.abort_flag)) return false;
        tg::tc_fence_after();
        const uint32_t k0 = tg::smem_u32(S.k[j & 1][0]);
#pragma unroll
        for (int kk = 4 * h; kk < 4 * h + 4; ++kk) {
          const uint64_t bdesc = tg::smem_desc_sw128(k0 + kk * 16 * 128, kBN * 64 * 2, 1024);
          tg::mma_bf16_ts(tmem + kColAcc, tmem + kColS + 64 * h + (kk - 4 * h) * 8, bdesc, idesc_q,
                          (j | kk) != 0);
        }
        if (h == 1) tg::mma_commit(&S.kv_empty[j & 1]);
        if (h == 1 && j == nt - 1) tg::mma_commit(&S.dq_done);
        return true;
      };
      if (alive) alive = issue_sp(0, 0) && issue_sp(0, 1);
      for (int j = 0; j < nt && alive; ++j) {
        alive = issue_dq(j, 0);
        if (alive && j + 1 < nt) alive = issue_sp(j + 1, 0);
        if (alive) alive = issue_dq(j, 1);
        if (alive && j + 1 < nt) alive = issue_sp(j + 1, 1);
      }
    }
    __syncwarp();
  } else if (warp == 6) {
    // ---- the key tiles' biases log2(e) g_h s_j ----
    const float g2 = gain[hq] * kLog2e;
    for (int j = 0; j < nt; ++j) {
      const int st = j & 1;
      if (j >= 2 && !__all_sync(0xFFFFFFFFu, tg::mbar_wait(&S.b_empty[st], ((j >> 1) - 1) & 1,
                                                           status, &S.abort_flag)))
        break;
#pragma unroll
      for (int u = 0; u < kBN / 32; ++u) {
        const int kp = j * kBN + lane + 32 * u;
        S.bias[st][lane + 32 * u] =
            kp < len && tg::in_bounds(seq0 + kp, total, status) ? g2 * s_kept[seq0 + kp] : 0.f;
      }
      tg::mbar_arrive(&S.b_full[st]);
    }
  } else if (warp < 4) {
    // ---- elementwise: dS = c_h P (dP - D), thread = query row (TMEM lane) ----
    const int r = warp * 32 + lane;
    const int qrow = t * kBM + r;
    const bool valid = qrow < len;
    const float th = tau[hq];
    const float c = 1.f / (sqrtf(static_cast<float>(kD)) * th);
    const float c2 = c * kLog2e;
    const float l2 = valid ? lse2[static_cast<int64_t>(hq) * total + seq0 + qrow] : 0.f;
    const float Dr = valid ? D[static_cast<int64_t>(hq) * total + seq0 + qrow] : 0.f;
    const uint32_t sa = tmem_lane_addr(tmem, warp, kColS), da = tmem_lane_addr(tmem, warp, kColDP);
    bool alive = true;
    for (int j = 0; j < nt && alive; ++j) {
      const int st = j & 1;
      alive = tg::mbar_wait(&S.b_full[st], (j >> 1) & 1, status, &S.abort_flag);
      const bool diag = (j == t);
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {   // 64-key halves, each as soon as its S and dP land
      if (alive) alive = tg::mbar_wait(&S.sp_full[h], j & 1, status, &S.abort_flag);
      if (!__all_sync(0xFFFFFFFFu, alive)) { alive = false; break; }
      tg::tc_fence_after();
#pragma unroll 1
      for (int ch = 2 * h; ch < 2 * h + 2; ++ch) {
        uint32_t sv[32], pv[32], pk[16];
        tg::tmem_ld32(sa + 32 * ch, sv);
        tg::tmem_ld32(da + 32 * ch, pv);
        tg::tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float d2[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int col = 32 * ch + e + u;
            float p = tg::exp2_approx(fmaf(__uint_as_float(sv[e + u]), c2, S.bias[st][col] - l2));
            if (!valid || (diag && col > r)) p = 0.f;
            d2[u] = p * (__uint_as_float(pv[e + u]) - Dr) * c;
          }
          pk[e / 2] = tg::pack_bf16x2(d2[0], d2[1]);
        }
        // packed columns 64h + 16(ch-2h) .. +15 of S, inside this half's own 64
        // columns (which this thread has read already)
        tg::tmem_st16(sa + 64 * h + 16 * (ch - 2 * h), pk);
      }
      tg::tmem_st_wait();
      tg::tc_fence_before();
      __syncwarp();
      if (lane == 0) tg::mbar_arrive(&S.ds_full[h]);
      }
      if (!alive) break;
      if (lane == 0) tg::mbar_arrive(&S.b_empty[st]);
    }
    if (alive) alive = tg::mbar_wait(&S.dq_done, 0, status, &S.abort_flag);
    if (__all_sync(0xFFFFFFFFu, alive)) {
      tg::tc_fence_after();
      const uint32_t qa = tmem_lane_addr(tmem, warp, kColAcc);
#pragma unroll 1
      for (int ch = 0; ch < kD / 32; ++ch) {
        uint32_t a[32];
        tg::tmem_ld32(qa + 32 * ch, a);
        tg::tmem_ld_wait();
        if (valid && tg::in_bounds(seq0 + qrow, total, status)) {
          uint4* dst = reinterpret_cast<uint4*>(
              dq + (static_cast<int64_t>(seq0 + qrow) * n_hq + hq) * kD + 32 * ch);
#pragma unroll
          for (int u = 0; u < 4; ++u)
            dst[u] = make_uint4(tg::pack_bf16x2(__uint_as_float(a[8 * u]), __uint_as_float(a[8 * u + 1])),
                                tg::pack_bf16x2(__uint_as_float(a[8 * u + 2]), __uint_as_float(a[8 * u + 3])),
                                tg::pack_bf16x2(__uint_as_float(a[8 * u + 4]), __uint_as_float(a[8 * u + 5])),
                                tg::pack_bf16x2(__uint_as_float(a[8 * u + 6]), __uint_as_float(a[8 * u + 7])));
        }
      }
    }
  }
  tg::tc_fence_before();
  __syncthreads();
  if (warp == 7) {
    tg::tc_fence_after();
    tg::tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------------- //
// bf16: dK, dV and the score / gain / temperature partials                   //
// ------------------------------------------------------------------------- //
struct DkvSmem {
  uint8_t k[2][kBN * 64 * 2];          // K_j (once)
  uint8_t v[2][kBN * 64 * 2];          // V_j (once)
  uint8_t q[2][2][kBM * 64 * 2];       // Q_i ring
  uint8_t dout[2][2][kBM * 64 * 2];    // dO_i ring
  float lse2[2][kBM];                  // the ring's query rows
  float D[2][kBM];
  uint64_t kv_full;
  uint64_t qd_full[2], qd_empty[2];
  uint64_t ld_full[2], ld_empty[2];
  uint64_t st_full[2], pd_full[2], acc_done;   // per 64-query half of the item
  uint32_t tmem_base;
  int abort_flag;
};
constexpr uint32_t kColST = 0, kColDPT = 128, kColDV = 256, kColDK = 384;

__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const float* __restrict__ s_kept, const float* __restrict__ gain,
                    const float* __restrict__ tau, const int32_t* __restrict__ cu_kept, int total,
                    int max_kept, int n_hq, int n_hkv, const float* __restrict__ D,
                    const float* __restrict__ lse2, int batch, int nsplit,
                    __nv_bfloat16* __restrict__ dk, __nv_bfloat16* __restrict__ dv,
                    float* __restrict__ dkv_part, float* __restrict__ ds_part,
                    float* __restrict__ gt_part, int* status) {
  // blockIdx.x = ((jt * batch + b) * n_hkv + kvh) * nsplit + half: key tile 0, which
  // meets the most query tiles, for every sequence and head first (longest first)
  const int cta = blockIdx.x;
  const int half = cta % nsplit;
  const int kvh = (cta / nsplit) % n_hkv;
  const int b = (cta / nsplit / n_hkv) % batch;
  const int jt = cta / nsplit / n_hkv / batch;
  const int G = n_hq / n_hkv;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (tg::smem_u32(smem_raw) & 1023u)) & 1023u;
  DkvSmem& S = *reinterpret_cast<DkvSmem*>(smem_raw + pad);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    tg::mbar_init(&S.kv_full, 1);
    for (int i = 0; i < 2; ++i) {
      tg::mbar_init(&S.qd_full[i], 1);
      tg::mbar_init(&S.qd_empty[i], 1);
      tg::mbar_init(&S.ld_full[i], 32);
      tg::mbar_init(&S.ld_empty[i], 4);
    }
    for (int i = 0; i < 2; ++i) {
      tg::mbar_init(&S.st_full[i], 1);
      tg::mbar_init(&S.pd_full[i], 4);
    }
    tg::mbar_init(&S.acc_done, 1);
    S.abort_flag = 0;
    tg::fence_barrier_init();
  }
  if (warp == 7) {
    tg::tmem_alloc(&S.tmem_base, 512);
    tg::tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    tg::tma_prefetch_desc(&tm_q);
    tg::tma_prefetch_desc(&tm_k);
    tg::tma_prefetch_desc(&tm_v);
    tg::tma_prefetch_desc(&tm_do);
  }
  tg::tc_fence_before();
  __syncthreads();
  tg::tc_fence_after();
  const uint32_t tmem = S.tmem_base;
  tg::pdl_launch_dependents();
  tg::pdl_wait();

  const int seq0 = cu_kept[b], seq1 = cu_kept[b + 1];
  const bool bad = seq0 < 0 || seq1 < seq0 || seq1 > total || seq1 - seq0 > max_kept;
  if (bad && kvh == 0 && jt == 0 && tid == 0) tg::set_status(status, TG_ERR_DEVICE_CHECK);
  const int len = bad ? 0 : seq1 - seq0;
  // the reduction reads every gain/temperature slot of every CTA: start at zero
  for (int e = tid; e < G * 4 * 2; e += kBwdThreads) gt_part[static_cast<int64_t>(cta) * G * 8 + e] = 0.f;
  if (jt * kBN >= len) {   // no key of this tile
    if (warp == 7) tg::tmem_dealloc(tmem, 512);
    return;
  }
  const int n_qt = (len + kBM - 1) / kBM;
  const int per_head = n_qt - jt;   // query tiles jt..n_qt-1
  const int n_all = G * per_head;   // (head, query tile) items of the unit, head-major
  const int it0 = n_all * half / nsplit, it1 = n_all * (half + 1) / nsplit;
  const int n_items = it1 - it0;    // this CTA's items it0 .. it1-1 (local index it - it0)
  // split units: this half's dK and dV partials, fp32 [total, n_hkv, dh] each
  float* const dk_part = dkv_part + static_cast<int64_t>(half * 2) * total * n_hkv * kD;
  float* const dv_part = dkv_part + static_cast<int64_t>(half * 2 + 1) * total * n_hkv * kD;
  __syncthreads();   // the slots are zero before any warp writes its own
  if (n_items == 0) {   // nothing to add: zero partials for this tile's keys
    if (warp < 4) {
      const int krow = jt * kBN + warp * 32 + lane;
      if (krow < len) {
        const int64_t o = (static_cast<int64_t>(seq0 + krow) * n_hkv + kvh) * kD;
        for (int d = 0; d < kD; d += 4) {
          *reinterpret_cast<float4*>(dk_part + o + d) = make_float4(0.f, 0.f, 0.f, 0.f);
          *reinterpret_cast<float4*>(dv_part + o + d) = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        ds_part[(static_cast<int64_t>(half) * n_hkv + kvh) * total + seq0 + krow] = 0.f;
      }
    }
    if (warp == 7) tg::tmem_dealloc(tmem, 512);
    return;
  }

  if (warp == 4) {
    // ---- TMA: K_j and V_j once, then the (Q_i, dO_i) ring ----
    if (lane == 0) {
      tg::mbar_arrive_expect_tx(&S.kv_full, 2 * kBN * kD * 2);
      for (int hh = 0; hh < 2; ++hh) {
        tg::tma_load_3d(S.k[hh], &tm_k, &S.kv_full, 64 * hh, kvh, seq0 + jt * kBN);
        tg::tma_load_3d(S.v[hh], &tm_v, &S.kv_full, 64 * hh, kvh, seq0 + jt * kBN);
      }
      int it = 0;
      for (; it < n_items; ++it) {
        const int st = it & 1;
        const int h = kvh * G + (it0 + it) / per_head, i = jt + (it0 + it) % per_head;
        if (it >= 2 && !tg::mbar_wait(&S.qd_empty[st], ((it >> 1) - 1) & 1, status, &S.abort_flag)) break;
        tg::mbar_arrive_expect_tx(&S.qd_full[st], 2 * kBM * kD * 2);
        for (int hh = 0; hh < 2; ++hh) {
          tg::tma_load_3d(S.q[st][hh], &tm_q, &S.qd_full[st], 64 * hh, h, seq0 + i * kBM);
          tg::tma_load_3d(S.dout[st][hh], &tm_do, &S.qd_full[st], 64 * hh, h, seq0 + i * kBM);
        }
      }
      if (S.abort_flag) {
        tg::mbar_wait(&S.kv_full, 0, status, nullptr);
        for (int i = it > 2 ? it - 2 : 0; i < it; ++i)
          tg::mbar_wait(&S.qd_full[i & 1], (i >> 1) & 1, status, nullptr);
      }
    }
    __syncwarp();
  } else if (warp == 5) {
    // ---- MMA: S^T = K Q^T, dP^T = V dO^T; then dV += P^T dO, dK += dS^T Q ----
    // By 64-query halves, in the order ST_lo dPT_lo, ST_hi dPT_hi, dV_lo dK_lo, (next
    // item) ST_lo dPT_lo, dV_hi dK_hi, ST_hi dPT_hi, ...: the elementwise warps work on
    // one half while the tensor core computes the other. A half's S^T and dP^T are
    // rewritten only after the dV/dK MMAs reading its P^T and dS^T were issued.
    if (lane == 0) {
      constexpr uint32_t idesc_h = tg::idesc_bf16_f32(kBN, kBM / 2, false, false);
      constexpr uint32_t idesc_o = tg::idesc_bf16_f32(kBN, kD, false, true);
      bool alive = tg::mbar_wait(&S.kv_full, 0, status, &S.abort_flag);
      const uint32_t k0 = tg::smem_u32(S.k[0]), v0 = tg::smem_u32(S.v[0]);
      // S^T and dP^T of half h of item it (queries 64h .. 64h+63: rows 64h of the
      // 128-byte-swizzled Q and dO tiles, 8 KB into each 64-dim half)
      auto issue_sp = [&](int it, int h) -> bool {
        const int st = it & 1;
        if (h == 0 && !tg::mbar_wait(&S.qd_full[st], (it >> 1) & 1, status, &S.abort_flag))
          return false;
        tg::tc_fence_after();
        const uint32_t q0 = tg::smem_u32(S.q[st][0]) + h * (kBM / 2) * 128;
        const uint32_t d0 = tg::smem_u32(S.dout[st][0]) + h * (kBM / 2) * 128;
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (kBM * 64 * 2) + (kk & 3) * 32;
          tg::mma_bf16_ss(tmem + kColST + 64 * h, tg::smem_desc_sw128(k0 + off, 16, 1024),
                          tg::smem_desc_sw128(q0 + off, 16, 1024), idesc_h, kk != 0);
        }
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (kBM * 64 * 2) + (kk & 3) * 32;
          tg::mma_bf16_ss(tmem + kColDPT + 64 * h, tg::smem_desc_sw128(v0 + off, 16, 1024),
                          tg::smem_desc_sw128(d0 + off, 16, 1024), idesc_h, kk != 0);
        }
        tg::mma_commit(&S.st_full[h]);
        return true;
      };
      // dV += P^T_h dO_h, dK += dS^T_h Q_h: A = the half's packed bf16 at columns
      // 64h .. 64h+31 (8 columns per 16 queries); B = dO_i / Q_i rows 64h + 16kk ..
      // as MN-major operands
      auto issue_acc = [&](int it, int h) -> bool {
        if (!tg::mbar_wait(&S.pd_full[h], it & 1, status, &S.abort_flag)) return false;
        tg::tc_fence_after();
        const int st = it & 1;
        const uint32_t q0 = tg::smem_u32(S.q[st][0]), d0 = tg::smem_u32(S.dout[st][0]);
#pragma unroll
        for (int kk = 4 * h; kk < 4 * h + 4; ++kk) {
          const uint32_t acc = (it | kk) != 0;
          const uint32_t a_col = 64 * h + (kk - 4 * h) * 8;
          tg::mma_bf16_ts(tmem + kColDV, tmem + kColST + a_col,
                          tg::smem_desc_sw128(d0 + kk * 16 * 128, kBM * 64 * 2, 1024), idesc_o, acc);
          tg::mma_bf16_ts(tmem + kColDK, tmem + kColDPT + a_col,
                          tg::smem_desc_sw128(q0 + kk * 16 * 128, kBM * 64 * 2, 1024), idesc_o, acc);
        }
        if (h == 1) tg::mma_commit(&S.qd_empty[st]);
        if (h == 1 && it == n_items - 1) tg::mma_commit(&S.acc_done);
        return true;
      };
      if (alive) alive = issue_sp(0, 0) && issue_sp(0, 1);
      for (int it = 0; it < n_items && alive; ++it) {
        alive = issue_acc(it, 0);
        if (alive && it + 1 < n_items) alive = issue_sp(it + 1, 0);
        if (alive) alive = issue_acc(it, 1);
        if (alive && it + 1 < n_items) alive = issue_sp(it + 1, 1);
      }
    }
    __syncwarp();
  } else if (warp == 6) {
    // ---- each item's query rows: lse2 and D (plain loads; row offsets are arbitrary) ----
    for (int it = 0; it < n_items; ++it) {
      const int st = it & 1;
      const int h = kvh * G + (it0 + it) / per_head, i = jt + (it0 + it) % per_head;
      if (it >= 2 && !__all_sync(0xFFFFFFFFu, tg::mbar_wait(&S.ld_empty[st], ((it >> 1) - 1) & 1,
                                                            status, &S.abort_flag)))
        break;
#pragma unroll
      for (int u = 0; u < kBM / 32; ++u) {
        const int qr = i * kBM + lane + 32 * u;
        const bool ok = qr < len;
        S.lse2[st][lane + 32 * u] = ok ? lse2[static_cast<int64_t>(h) * total + seq0 + qr] : 0.f;
        S.D[st][lane + 32 * u] = ok ? D[static_cast<int64_t>(h) * total + seq0 + qr] : 0.f;
      }
      tg::mbar_arrive(&S.ld_full[st]);
    }
  } else if (warp < 4) {
    // ---- elementwise: thread = key row (TMEM lane) ----
    const int r = warp * 32 + lane;
    const int krow = jt * kBN + r;
    const bool kvalid = krow < len;
    const float sk = kvalid && tg::in_bounds(seq0 + krow, total, status) ? s_kept[seq0 + krow] : 0.f;
    const uint32_t sa = tmem_lane_addr(tmem, warp, kColST), da = tmem_lane_addr(tmem, warp, kColDPT);
    float ds_acc = 0.f;      // sum_h g_h sum_i dZ for this key
    float dz_h = 0.f, tz_h = 0.f;   // this head's sum_i dZ and sum_i dZ (q.k)
    bool alive = true;
    for (int it = 0; it < n_items; ++it) {
      const int st = it & 1;
      const int hl = (it0 + it) / per_head, h = kvh * G + hl, i = jt + (it0 + it) % per_head;
      const float th = tau[h];
      const float c = 1.f / (sqrtf(static_cast<float>(kD)) * th);
      const float c2 = c * kLog2e;
      const float b2 = gain[h] * kLog2e * sk;
      alive = tg::mbar_wait(&S.ld_full[st], (it >> 1) & 1, status, &S.abort_flag);
      const bool diag = (i == jt);
      const int qlim = len - i * kBM;   // query rows of this tile inside the sequence
#pragma unroll 1
      for (int hq2 = 0; hq2 < 2; ++hq2) {   // 64-query halves, each as its S^T and dP^T land
      if (alive) alive = tg::mbar_wait(&S.st_full[hq2], it & 1, status, &S.abort_flag);
      if (!__all_sync(0xFFFFFFFFu, alive)) { alive = false; break; }
      tg::tc_fence_after();
#pragma unroll 1
      for (int ch = 2 * hq2; ch < 2 * hq2 + 2; ++ch) {
        uint32_t sv[32], pv[32], pp[16], pd[16];
        tg::tmem_ld32(sa + 32 * ch, sv);
        tg::tmem_ld32(da + 32 * ch, pv);
        tg::tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float p2[2], d2[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int col = 32 * ch + e + u;   // query row i*128 + col
            const float sr = __uint_as_float(sv[e + u]);
            float p = tg::exp2_approx(fmaf(sr, c2, b2 - S.lse2[st][col]));
            // key after the query, or key or query past the sequence's end
            if (!kvalid || col >= qlim || (diag && r > col)) p = 0.f;
            const float dz = p * (__uint_as_float(pv[e + u]) - S.D[st][col]);
            dz_h += dz;
            tz_h = fmaf(dz, sr, tz_h);
            p2[u] = p;
            d2[u] = dz * c;
          }
          pp[e / 2] = tg::pack_bf16x2(p2[0], p2[1]);
          pd[e / 2] = tg::pack_bf16x2(d2[0], d2[1]);
        }
        // packed columns 64h + 16(ch-2h) .. +15 of S^T / dP^T, inside this half's
        // own 64 columns (which this thread has read already)
        tg::tmem_st16(sa + 64 * hq2 + 16 * (ch - 2 * hq2), pp);
        tg::tmem_st16(da + 64 * hq2 + 16 * (ch - 2 * hq2), pd);
      }
      tg::tmem_st_wait();
      tg::tc_fence_before();
      __syncwarp();
      if (lane == 0) tg::mbar_arrive(&S.pd_full[hq2]);
      }
      if (!alive) break;
      if (lane == 0) tg::mbar_arrive(&S.ld_empty[st]);
      if ((it0 + it) % per_head == per_head - 1 || it == n_items - 1) {
        // this head's items in this CTA are done: its score-gradient share, and this
        // warp's gain and temperature partials for it (summed over the CTA's warps and
        // the unit's two CTAs by the reduction, so no barrier between warps is needed)
        ds_acc = fmaf(gain[h], dz_h, ds_acc);
        float gsum = dz_h * sk, tsum = tz_h;
        for (int off = 16; off > 0; off >>= 1) {
          gsum += __shfl_xor_sync(0xFFFFFFFFu, gsum, off);
          tsum += __shfl_xor_sync(0xFFFFFFFFu, tsum, off);
        }
        if (lane == 0) {
          float* gp = gt_part + ((static_cast<int64_t>(cta) * G + hl) * 4 + warp) * 2;
          gp[0] = gsum;
          gp[1] = -(c / th) * tsum;
        }
        dz_h = 0.f;
        tz_h = 0.f;
      }
    }
    if (kvalid && alive && tg::in_bounds(seq0 + krow, total, status))
      ds_part[(static_cast<int64_t>(half) * n_hkv + kvh) * total + seq0 + krow] = ds_acc;
    if (alive) alive = tg::mbar_wait(&S.acc_done, 0, status, &S.abort_flag);
    if (__all_sync(0xFFFFFFFFu, alive)) {
      tg::tc_fence_after();
#pragma unroll 1
      for (int which = 0; which < 2; ++which) {
        const uint32_t aa = tmem_lane_addr(tmem, warp, which ? kColDK : kColDV);
        float* dst_base = which ? dk_part : dv_part;
        __nv_bfloat16* out_base = which ? dk : dv;
#pragma unroll 1
        for (int ch = 0; ch < kD / 32; ++ch) {
          uint32_t a[32];
          tg::tmem_ld32(aa + 32 * ch, a);
          tg::tmem_ld_wait();
          if (kvalid && !tg::in_bounds(seq0 + krow, total, status)) {
            // debug library: a row outside the kept rows is not written
          } else if (kvalid && nsplit == 1) {   // the whole unit: dK, dV rows in bf16
            uint4* dst = reinterpret_cast<uint4*>(
                out_base + (static_cast<int64_t>(seq0 + krow) * n_hkv + kvh) * kD + 32 * ch);
#pragma unroll
            for (int u = 0; u < 4; ++u)
              dst[u] = make_uint4(tg::pack_bf16x2(__uint_as_float(a[8 * u]), __uint_as_float(a[8 * u + 1])),
                                  tg::pack_bf16x2(__uint_as_float(a[8 * u + 2]), __uint_as_float(a[8 * u + 3])),
                                  tg::pack_bf16x2(__uint_as_float(a[8 * u + 4]), __uint_as_float(a[8 * u + 5])),
                                  tg::pack_bf16x2(__uint_as_float(a[8 * u + 6]), __uint_as_float(a[8 * u + 7])));
          } else if (kvalid) {
            float4* dst = reinterpret_cast<float4*>(
                dst_base + (static_cast<int64_t>(seq0 + krow) * n_hkv + kvh) * kD + 32 * ch);
#pragma unroll
            for (int u = 0; u < 8; ++u)
              dst[u] = make_float4(__uint_as_float(a[4 * u]), __uint_as_float(a[4 * u + 1]),
                                   __uint_as_float(a[4 * u + 2]), __uint_as_float(a[4 * u + 3]));
          }
        }
      }
    }
  }
  tg::tc_fence_before();
  __syncthreads();
  if (warp == 7) {
    tg::tc_fence_after();
    tg::tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------------- //
// f32 (exact SIMT, small problems)                                           //
// ------------------------------------------------------------------------- //
constexpr int kF32MaxPerLane = 8;   // dh <= 256

__device__ __forceinline__ int seq_of(const int32_t* cu, int batch, int64_t row) {
  int b = 0;
  while (b + 1 < batch && cu[b + 1] <= row) ++b;
  return b;
}

__device__ __forceinline__ float warp_sum(float v) {
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, off);
  return v;
}

// one warp per (query row i, head): dq_i = c sum_j dZ_ij k_j
__global__ void __launch_bounds__(128)
    bwd_f32_dq_kernel(const float* __restrict__ q, const float* __restrict__ k,
                      const float* __restrict__ v, const float* __restrict__ dout,
                      const float* __restrict__ s_kept, const float* __restrict__ gain,
                      const float* __restrict__ tau, const int32_t* __restrict__ cu_kept, int batch,
                      int64_t total, int n_hq, int n_hkv, int dh, const float* __restrict__ D,
                      const float* __restrict__ lse2, float* __restrict__ dq, int* status) {
  tg::pdl_launch_dependents();
  tg::pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t i = static_cast<int64_t>(blockIdx.x) * 4 + (threadIdx.x >> 5);
  const int h = blockIdx.y;
  if (i >= total) return;
  const int b = seq_of(cu_kept, batch, i);
  const int64_t j0 = cu_kept[b];
  if (j0 < 0 || j0 > i) {
    if (lane == 0) tg::set_status(status, TG_ERR_DEVICE_CHECK);
    return;
  }
  const int kv = h / (n_hq / n_hkv);
  const float c = 1.f / (sqrtf(static_cast<float>(dh)) * tau[h]);
  const float g = gain[h];
  const float l2 = lse2[static_cast<int64_t>(h) * total + i];
  const float Di = D[static_cast<int64_t>(h) * total + i];
  float qv[kF32MaxPerLane], dov[kF32MaxPerLane], acc[kF32MaxPerLane];
#pragma unroll
  for (int e = 0; e < kF32MaxPerLane; ++e) {
    const int col = lane + 32 * e;
    qv[e] = col < dh ? q[(i * n_hq + h) * dh + col] : 0.f;
    dov[e] = col < dh ? dout[(i * n_hq + h) * dh + col] : 0.f;
    acc[e] = 0.f;
  }
  for (int64_t j = j0; j <= i; ++j) {
    if (!tg::in_bounds(j, total, status)) break;
    const float* kj = k + (j * n_hkv + kv) * dh;
    const float* vj = v + (j * n_hkv + kv) * dh;
    float qk = 0.f, dp = 0.f;
#pragma unroll
    for (int e = 0; e < kF32MaxPerLane; ++e) {
      const int col = lane + 32 * e;
      if (col < dh) {
        qk = fmaf(qv[e], kj[col], qk);
        dp = fmaf(dov[e], vj[col], dp);
      }
    }
    qk = warp_sum(qk);
    dp = warp_sum(dp);
    const float p = exp2f((c * qk + g * s_kept[j]) * kLog2e - l2);
    const float dz = p * (dp - Di);
#pragma unroll
    for (int e = 0; e < kF32MaxPerLane; ++e) {
      const int col = lane + 32 * e;
      if (col < dh) acc[e] = fmaf(c * dz, kj[col], acc[e]);
    }
  }
#pragma unroll
  for (int e = 0; e < kF32MaxPerLane; ++e) {
    const int col = lane + 32 * e;
    if (col < dh) dq[(i * n_hq + h) * dh + col] = acc[e];
  }
}

// one warp per (key j, KV head): dk_j, dv_j, the score-gradient share and the
// gain / temperature partials of every head of the group (per key, per head)
__global__ void __launch_bounds__(128)
    bwd_f32_dkdv_kernel(const float* __restrict__ q, const float* __restrict__ k,
                        const float* __restrict__ v, const float* __restrict__ dout,
                        const float* __restrict__ s_kept, const float* __restrict__ gain,
                        const float* __restrict__ tau, const int32_t* __restrict__ cu_kept,
                        int batch, int64_t total, int n_hq, int n_hkv, int dh,
                        const float* __restrict__ D, const float* __restrict__ lse2,
                        float* __restrict__ dk, float* __restrict__ dv,
                        float* __restrict__ ds_part, float* __restrict__ gt_row, int* status) {
  tg::pdl_launch_dependents();
  tg::pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t j = static_cast<int64_t>(blockIdx.x) * 4 + (threadIdx.x >> 5);
  const int kv = blockIdx.y;
  if (j >= total) return;
  const int b = seq_of(cu_kept, batch, j);
  const int64_t i1 = cu_kept[b + 1];
  if (i1 <= j || i1 > total) {
    if (lane == 0) tg::set_status(status, TG_ERR_DEVICE_CHECK);
    return;
  }
  const int G = n_hq / n_hkv;
  float kvv[kF32MaxPerLane], vvv[kF32MaxPerLane], ak[kF32MaxPerLane], av[kF32MaxPerLane];
#pragma unroll
  for (int e = 0; e < kF32MaxPerLane; ++e) {
    const int col = lane + 32 * e;
    kvv[e] = col < dh ? k[(j * n_hkv + kv) * dh + col] : 0.f;
    vvv[e] = col < dh ? v[(j * n_hkv + kv) * dh + col] : 0.f;
    ak[e] = av[e] = 0.f;
  }
  const float sj = s_kept[j];
  float ds_acc = 0.f;
  for (int hl = 0; hl < G; ++hl) {
    const int h = kv * G + hl;
    const float th = tau[h];
    const float c = 1.f / (sqrtf(static_cast<float>(dh)) * th);
    const float g = gain[h];
    float dzs = 0.f, tzs = 0.f;
    for (int64_t i = j; i < i1; ++i) {
      if (!tg::in_bounds(i, total, status)) break;
      const float* qi = q + (i * n_hq + h) * dh;
      const float* di = dout + (i * n_hq + h) * dh;
      float qk = 0.f, dp = 0.f;
#pragma unroll
      for (int e = 0; e < kF32MaxPerLane; ++e) {
        const int col = lane + 32 * e;
        if (col < dh) {
          qk = fmaf(qi[col], kvv[e], qk);
          dp = fmaf(di[col], vvv[e], dp);
        }
      }
      qk = warp_sum(qk);
      dp = warp_sum(dp);
      const float p = exp2f((c * qk + g * sj) * kLog2e - lse2[static_cast<int64_t>(h) * total + i]);
      const float dz = p * (dp - D[static_cast<int64_t>(h) * total + i]);
      dzs += dz;
      tzs = fmaf(dz, qk, tzs);
#pragma unroll
      for (int e = 0; e < kF32MaxPerLane; ++e) {
        const int col = lane + 32 * e;
        if (col < dh) {
          ak[e] = fmaf(c * dz, qi[col], ak[e]);
          av[e] = fmaf(p, di[col], av[e]);
        }
      }
    }
    ds_acc = fmaf(g, dzs, ds_acc);
    if (lane == 0) {
      gt_row[(j * n_hq + h) * 2] = dzs * sj;
      gt_row[(j * n_hq + h) * 2 + 1] = -(c / th) * tzs;
    }
  }
#pragma unroll
  for (int e = 0; e < kF32MaxPerLane; ++e) {
    const int col = lane + 32 * e;
    if (col < dh) {
      dk[(j * n_hkv + kv) * dh + col] = ak[e];
      dv[(j * n_hkv + kv) * dh + col] = av[e];
    }
  }
  if (lane == 0) ds_part[static_cast<int64_t>(kv) * total + j] = ds_acc;
}

// ------------------------------------------------------------------------- //
// reductions (fixed order)                                                   //
// ------------------------------------------------------------------------- //
// ds_j = sum over KV heads of the per-KV-head shares
__global__ void __launch_bounds__(256)
    bwd_reduce_ds_kernel(const float* __restrict__ ds_part, int64_t total, int n_hkv,
                         float* __restrict__ ds) {
  tg::pdl_launch_dependents();
  tg::pdl_wait();
  const int64_t j = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
  if (j >= total) return;
  float a = 0.f;
  for (int kv = 0; kv < n_hkv; ++kv) a += ds_part[static_cast<int64_t>(kv) * total + j];
  ds[j] = a;
}

// bf16 path: for each key row of a valid sequence, ds = the sum over halves and KV
// heads of the shares and, for split units, dK and dV = half 0 + half 1 of the
// partials, in that fixed order. Rows of a sequence that failed the device check are
// left alone (their partials were never written). One warp per (key row, KV head)
// for split units, one per key row otherwise.
__global__ void __launch_bounds__(256)
    bwd_reduce_dkv_ds_kernel(const float* __restrict__ dkv_part, const float* __restrict__ ds_part,
                             const int32_t* __restrict__ cu_kept, int batch, int64_t total,
                             int max_kept, int n_hkv, int nsplit, __nv_bfloat16* __restrict__ dk,
                             __nv_bfloat16* __restrict__ dv, float* __restrict__ ds) {
  tg::pdl_launch_dependents();
  tg::pdl_wait();
  // split units: one warp per (row j, KV head kv), its four 512-byte loads all in
  // flight at once; whole units: one warp per row (the score gradient only)
  const int per_row = nsplit > 1 ? n_hkv : 1;
  const int64_t w = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int64_t j = w / per_row;
  const int kv = static_cast<int>(w % per_row);
  const int lane = threadIdx.x & 31;
  if (j >= total) return;
  int lo = 0, hi = batch;   // the sequence holding row j: cu_kept[b] <= j < cu_kept[b + 1]
  while (hi - lo > 1) {
    const int mid = (lo + hi) / 2;
    if (cu_kept[mid] <= j) lo = mid;
    else hi = mid;
  }
  const int64_t s0 = cu_kept[lo], s1 = cu_kept[lo + 1];
  if (s0 < 0 || s1 < s0 || s1 > total || s1 - s0 > max_kept || j < s0 || j >= s1) return;
  const int64_t plane = total * n_hkv * kD;
  if (nsplit > 1) {
    const int64_t o = (j * n_hkv + kv) * kD + 4 * lane;
    const float4 k0 = *reinterpret_cast<const float4*>(dkv_part + o);
    const float4 v0 = *reinterpret_cast<const float4*>(dkv_part + plane + o);
    const float4 k1 = *reinterpret_cast<const float4*>(dkv_part + 2 * plane + o);
    const float4 v1 = *reinterpret_cast<const float4*>(dkv_part + 3 * plane + o);
    *reinterpret_cast<uint2*>(dk + o) =
        make_uint2(tg::pack_bf16x2(k0.x + k1.x, k0.y + k1.y), tg::pack_bf16x2(k0.z + k1.z, k0.w + k1.w));
    *reinterpret_cast<uint2*>(dv + o) =
        make_uint2(tg::pack_bf16x2(v0.x + v1.x, v0.y + v1.y), tg::pack_bf16x2(v0.z + v1.z, v0.w + v1.w));
  }
  if (kv == 0 && lane == 0) {   // the row's score gradient, in a fixed order
    float a = 0.f;
    for (int h2 = 0; h2 < nsplit; ++h2)
      for (int h = 0; h < n_hkv; ++h) a += ds_part[(static_cast<int64_t>(h2) * n_hkv + h) * total + j];
    ds[j] = a;
  }
}

// one block per query head: dg_h and dtau_h summed over the partials in a fixed
// order. Partials are [n_units][unit_heads][W][2]: bf16, a unit is a dK/dV CTA
// (b, kvh, key tile), its heads are the group's and W = 4 (one per elementwise
// warp); f32, a unit is a key row, its heads are all n_hq and W = 1.
__global__ void __launch_bounds__(256)
    bwd_reduce_gt_kernel(const float* __restrict__ part, int64_t n_units, int unit_heads, int W,
                         int units_per_group, int n_hq, int group, float* __restrict__ dgain,
                         float* __restrict__ dtau) {
  __shared__ float red[2][8];
  tg::pdl_launch_dependents();
  tg::pdl_wait();
  const int h = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float a = 0.f, t = 0.f;
  // bf16 partials: unit = CTA (b, kvh, jt), entries = the group's heads; f32
  // partials: unit = key row, entries = all heads (group ignored)
  for (int64_t u = threadIdx.x; u < n_units; u += 256) {
    int idx;
    if (units_per_group > 0) {   // CTA units: only those of head h's KV head
      const int64_t kvh_of_unit = (u / units_per_group) % (n_hq / group);
      if (kvh_of_unit != h / group) continue;
      idx = h % group;
    } else {
      idx = h;
    }
    for (int w = 0; w < W; ++w) {
      a += part[((u * unit_heads + idx) * W + w) * 2];
      t += part[((u * unit_heads + idx) * W + w) * 2 + 1];
    }
  }
  for (int off = 16; off > 0; off >>= 1) {
    a += __shfl_xor_sync(0xFFFFFFFFu, a, off);
    t += __shfl_xor_sync(0xFFFFFFFFu, t, off);
  }
  if (lane == 0) {
    red[0][warp] = a;
    red[1][warp] = t;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float sa = 0.f, st = 0.f;
    for (int w = 0; w < 8; ++w) {
      sa += red[0][w];
      st += red[1][w];
    }
    dgain[h] = sa;
    dtau[h] = st;
  }
}

size_t ws_bytes(int batch, int64_t total, int max_kept, int n_hq, int n_hkv, int head_dim,
                tg_dtype dt, BwdWs* ws, uint8_t* base) {
  // D and lse2 [n_hq, total]; ds partials [n_hkv, total]; gain/temperature
  // partials: bf16 per CTA and group head, f32 per key and head
  const int n_kt = (max_kept + kBN - 1) / kBN;
  const int G = n_hkv > 0 ? n_hq / n_hkv : 0;
  const bool bf = dt == TG_BF16;
  const int ns = bf ? kv_split(static_cast<int64_t>(n_kt) * batch * n_hkv) : 1;
  const int64_t gt = bf ? static_cast<int64_t>(n_kt) * ns * n_hkv * batch * G * 4 * 2
                        : total * n_hq * 2;
  const int64_t floats[5] = {n_hq * total, n_hq * total, ns * n_hkv * total, gt,
                             ns > 1 ? static_cast<int64_t>(ns) * 2 * total * n_hkv * kD : 0};
  size_t off = 0;
  float* ptrs[5];
  for (int i = 0; i < 5; ++i) {
    ptrs[i] = base ? reinterpret_cast<float*>(base + off) : nullptr;
    off += (static_cast<size_t>(floats[i]) * 4 + 255) / 256 * 256;
  }
  (void)head_dim;
  if (ws) *ws = BwdWs{ptrs[0], ptrs[1], ptrs[2], ptrs[3], ptrs[4]};
  return off;
}

}  // namespace

extern "C" size_t tg_gated_attention_bwd_workspace_size(tg_dtype dtype, int batch,
                                                        int64_t total_kept, int max_kept,
                                                        int n_hq, int n_hkv, int head_dim) {
  if (batch <= 0 || total_kept <= 0 || max_kept <= 0 || n_hq <= 0 || n_hkv <= 0 ||
      n_hq % n_hkv != 0 || head_dim <= 0)
    return 0;
  return ws_bytes(batch, total_kept, max_kept, n_hq, n_hkv, head_dim, dtype, nullptr, nullptr);
}

extern "C" tg_status tg_gated_attention_bwd(
    const void* q, const void* k, const void* v, const void* out, const void* dout,
    tg_dtype dtype, const float* lse, const float* s_kept, const float* gain, const float* tau,
    const int32_t* cu_kept, int batch, int64_t total_kept, int max_kept, int n_hq, int n_hkv,
    int head_dim, void* dq, void* dk, void* dv, float* ds, float* dgain, float* dtau,
    void* workspace, size_t workspace_bytes, tg_stream_t stream) {
  tg::NvtxRange nvtx_range("tg_gated_attention_bwd");
  if (batch < 0 || total_kept < 0 || max_kept < 0 || n_hq <= 0 || n_hkv <= 0 || head_dim <= 0)
    return TG_ERR_INVALID_ARG;
  if (batch == 0 || total_kept == 0 || max_kept == 0) return TG_OK;
  if (!q || !k || !v || !out || !dout || !lse || !s_kept || !gain || !tau || !cu_kept || !dq ||
      !dk || !dv || !ds || !dgain || !dtau)
    return TG_ERR_INVALID_ARG;
  if (n_hq % n_hkv != 0 || max_kept > total_kept) return TG_ERR_INVALID_ARG;
  if (n_hq > 65535 || n_hkv > 65535 || batch > 65535) return TG_ERR_UNSUPPORTED;
  if (dtype != TG_BF16 && dtype != TG_F32) return TG_ERR_UNSUPPORTED;
  if (dtype == TG_BF16 && head_dim != kD) return TG_ERR_UNSUPPORTED;
  if (dtype == TG_F32 && head_dim > 32 * kF32MaxPerLane) return TG_ERR_UNSUPPORTED;
  if (total_kept > INT32_MAX - kBM) return TG_ERR_UNSUPPORTED;
  BwdWs ws{};
  const size_t need = ws_bytes(batch, total_kept, max_kept, n_hq, n_hkv, head_dim, dtype, &ws,
                               static_cast<uint8_t*>(workspace));
  if (!workspace || workspace_bytes < need) return TG_ERR_WORKSPACE;
  if (!tg::aligned16(workspace)) return TG_ERR_MISALIGNED;
  if (dtype == TG_BF16 && (!tg::aligned16(q) || !tg::aligned16(k) || !tg::aligned16(v) ||
                           !tg::aligned16(dout) || !tg::aligned16(dq) || !tg::aligned16(dk) ||
                           !tg::aligned16(dv)))
    return TG_ERR_MISALIGNED;
  int* st = tg::status_word();
  if (!st) return TG_ERR_CUDA;
  const int G = n_hq / n_hkv;
  const int64_t prep_blocks = (total_kept * n_hq * 32 + 255) / 256;
  if (prep_blocks > INT32_MAX) return TG_ERR_UNSUPPORTED;
  tg_status r;
  if (dtype == TG_BF16) {
    r = tg::launch(bwd_prep_kernel<__nv_bfloat16>, dim3(static_cast<unsigned>(prep_blocks)), dim3(256),
                   0, stream, 0, static_cast<const __nv_bfloat16*>(out),
                   static_cast<const __nv_bfloat16*>(dout), lse, total_kept, n_hq, head_dim, ws.D,
                   ws.lse2);
    if (r != TG_OK) return r;
    CUtensorMap tq, tk, tv, tdo;
    const uint64_t dq_[3] = {kD, static_cast<uint64_t>(n_hq), static_cast<uint64_t>(total_kept)};
    const uint64_t sq_[2] = {kD * 2, static_cast<uint64_t>(n_hq) * kD * 2};
    const uint64_t dk_[3] = {kD, static_cast<uint64_t>(n_hkv), static_cast<uint64_t>(total_kept)};
    const uint64_t sk_[2] = {kD * 2, static_cast<uint64_t>(n_hkv) * kD * 2};
    const uint32_t box[3] = {64, 1, kBM};
    if (!tg::encode_tmap(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, q, dq_, sq_, box, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !tg::encode_tmap(&tdo, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, dout, dq_, sq_, box, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !tg::encode_tmap(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, k, dk_, sk_, box, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !tg::encode_tmap(&tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, v, dk_, sk_, box, CU_TENSOR_MAP_SWIZZLE_128B))
      return TG_ERR_CUDA;
    const int n_t = (max_kept + kBM - 1) / kBM;
    const size_t smem_dq = sizeof(DqSmem) + 1024, smem_kv = sizeof(DkvSmem) + 1024;
    if (!tg::ensure_smem(reinterpret_cast<const void*>(bwd_dq_kernel), static_cast<int>(smem_dq)) ||
        !tg::ensure_smem(reinterpret_cast<const void*>(bwd_dkdv_kernel), static_cast<int>(smem_kv)))
      return TG_ERR_CUDA;
    r = tg::launch(bwd_dq_kernel, dim3(n_hq, n_t, batch), dim3(kBwdThreads), smem_dq, stream, 0, tq,
                   tk, tv, tdo, s_kept, gain, tau, cu_kept, static_cast<int>(total_kept), max_kept,
                   n_hq, n_hkv, static_cast<const float*>(ws.D), static_cast<const float*>(ws.lse2),
                   static_cast<__nv_bfloat16*>(dq), st);
    if (r != TG_OK) return r;
    const int64_t units = static_cast<int64_t>(n_t) * batch * n_hkv;
    const int nsplit = kv_split(units);
    const int64_t kv_ctas = units * nsplit;
    if (kv_ctas > INT32_MAX) return TG_ERR_UNSUPPORTED;
    r = tg::launch(bwd_dkdv_kernel, dim3(static_cast<unsigned>(kv_ctas)), dim3(kBwdThreads), smem_kv,
                   stream, 0, tq, tk, tv, tdo, s_kept, gain, tau, cu_kept,
                   static_cast<int>(total_kept), max_kept, n_hq, n_hkv,
                   static_cast<const float*>(ws.D), static_cast<const float*>(ws.lse2), batch,
                   nsplit, static_cast<__nv_bfloat16*>(dk), static_cast<__nv_bfloat16*>(dv), ws.dkv,
                   ws.ds, ws.gt, st);
    if (r != TG_OK) return r;
    r = tg::launch(bwd_reduce_dkv_ds_kernel,
                   dim3(static_cast<unsigned>((total_kept * (nsplit > 1 ? n_hkv : 1) + 7) / 8)),
                   dim3(256), 0, stream, 0, static_cast<const float*>(ws.dkv),
                   static_cast<const float*>(ws.ds), cu_kept, batch, total_kept, max_kept, n_hkv,
                   nsplit, static_cast<__nv_bfloat16*>(dk), static_cast<__nv_bfloat16*>(dv), ds);
    if (r != TG_OK) return r;
    // CTA units ((jt, b, kvh), half): units_per_group = nsplit (a unit's CTAs share a KV head)
    return tg::launch(bwd_reduce_gt_kernel, dim3(n_hq), dim3(256), 0, stream, 0,
                      static_cast<const float*>(ws.gt), kv_ctas, G, 4, nsplit, n_hq, G, dgain,
                      dtau);
  }
  // f32
  r = tg::launch(bwd_prep_kernel<float>, dim3(static_cast<unsigned>(prep_blocks)), dim3(256), 0,
                 stream, 0, static_cast<const float*>(out), static_cast<const float*>(dout), lse,
                 total_kept, n_hq, head_dim, ws.D, ws.lse2);
  if (r != TG_OK) return r;
  const int64_t wblocks = (total_kept + 3) / 4;
  if (wblocks > INT32_MAX) return TG_ERR_UNSUPPORTED;
  r = tg::launch(bwd_f32_dq_kernel, dim3(static_cast<unsigned>(wblocks), n_hq), dim3(128), 0, stream,
                 0, static_cast<const float*>(q), static_cast<const float*>(k),
                 static_cast<const float*>(v), static_cast<const float*>(dout), s_kept, gain, tau,
                 cu_kept, batch, total_kept, n_hq, n_hkv, head_dim, static_cast<const float*>(ws.D),
                 static_cast<const float*>(ws.lse2), static_cast<float*>(dq), st);
  if (r != TG_OK) return r;
  r = tg::launch(bwd_f32_dkdv_kernel, dim3(static_cast<unsigned>(wblocks), n_hkv), dim3(128), 0,
                 stream, 0, static_cast<const float*>(q), static_cast<const float*>(k),
                 static_cast<const float*>(v), static_cast<const float*>(dout), s_kept, gain, tau,
                 cu_kept, batch, total_kept, n_hq, n_hkv, head_dim, static_cast<const float*>(ws.D),
                 static_cast<const float*>(ws.lse2), static_cast<float*>(dk),
                 static_cast<float*>(dv), ws.ds, ws.gt, st);
  if (r != TG_OK) return r;
  r = tg::launch(bwd_reduce_ds_kernel, dim3(static_cast<unsigned>((total_kept + 255) / 256)),
                 dim3(256), 0, stream, 0, static_cast<const float*>(ws.ds), total_kept, n_hkv, ds);
  if (r != TG_OK) return r;
  // key-row units: every head's entry in each unit
  return tg::launch(bwd_reduce_gt_kernel, dim3(n_hq), dim3(256), 0, stream, 0,
                    static_cast<const float*>(ws.gt), total_kept, n_hq, 1, 0, n_hq, G, dgain, dtau);
}

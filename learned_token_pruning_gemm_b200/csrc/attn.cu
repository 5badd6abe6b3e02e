// tg_gated_attention: token-gated causal GQA attention over the kept tokens
// (MarkTechPost page on TokenGate, section "Qu'est-ce que l'attention gérée par
// des tokens ?": each kept token's score is a bias on the attention logits,
// scaled by a learnable per-head gain; a learnable per-head temperature corrects
// for each query seeing fewer keys).
//     z_ij = q_i . k_j / (sqrt(dh) tau_h) + g_h s_j,  j <= i;  O_i = softmax_j(z) V
//
// bf16 path (dh = 128). Causal work grows with the query tile index t (tile t
// meets t+1 key tiles). One CTA per SM walks a list of query tiles: the (tile,
// sequence, head) items numbered longest tile first and dealt to the CTAs as a snake
// (c, 2G-1-c, 2G+c, ...), so every CTA's list sums to about the same number of key
// tiles and no CTA carries more than the longest tile plus what balances it; each
// next tile's loads and first S MMAs run under the tail of the one before (a CTA
// per tile paid ~4 us of start-up each, and pairs of tiles t, n-1-t per CTA left
// the longest tile's CTA one tile and one epilogue more than it needs).
// Per CTA, pipelines run across its query tiles:
//   warp 0       TMA producer of Q and of K tiles (128 keys) through a 3-stage
//                ring. A K stage is free as soon as S_j is computed; with S issued
//                three tiles ahead, each K load has about three tile periods to land.
//   warp 2       allocates TMEM, then stages each tile's per-key bias
//                b_j = log2(e) g_h s_j in a 4-stage ring of its own (so the K ring
//                never waits for the softmax to read a bias).
//   warp 3       TMA producer of V tiles through a 2-stage ring (free after PV_j).
//   warp 1       MMA issuer (one thread), order S_0, S_1, S_2, PV_0, S_3, PV_1,
//                S_4, ...: S_j = Q K_j^T into one of three 128-column TMEM buffers,
//                and O += P_j V_j with P_j read from TMEM (it overwrites S_j in
//                place) and V_j as an MN-major shared-memory operand. S_{j+3} reuses
//                the buffer of P_j right after PV_j, so the next two S tiles are
//                already computed whenever a softmax pass ends.
//   warps 4-11   softmax, one warp per 16 query rows (TMEM lane = row). S is read
//                in the 16x256b shape, which puts a row's 128 keys in one quad of
//                four threads (two rows per thread, 64 values), so row maxima and
//                sums are warp shuffles with no exchange between warps:
//                z = S c_h + b_j in the log2 domain (packed f32x2 FMA,
//                c_h = log2(e) / (sqrt(dh) tau_h)), diagonal-tile mask, a running
//                max that moves only when it grows by more than 2^8 (O is then
//                rescaled in TMEM), exp2 on the MUFU pipe for 3 of every 4 keys and
//                on the FMA pipe (own polynomial) for the 4th, P packed to bf16 and
//                written over S in the 16x128b shape (the A-operand layout of PV).
// Because P_j lives in S_j's buffer, softmax(j+1) runs while the tensor core does
// PV_j and S_{j+3}; the only cross-tile waits are the rare O rescale and, between
// the two query tiles, the epilogue's read of O before it is overwritten.
// P_j is reported on p_full[j % 3] and PV_j completes on o_done[j % 3]. Softmax
// warps run up to two tiles apart, each bounded by what it has seen: a warp that
// has seen S_j knows PV_{j-3} complete (S_j was issued after it), hence phase j-3 of
// p_full[j % 3] too, so its arrival for tile j counts toward tile j; and PV_{j+1}
// cannot start before the warp's own P_{j+1}, so at tile j the barrier that holds
// PV_{j-1} is at most one phase short of it and a parity wait on it is exact.
//
// f32 path: exact fp32 SIMT kernel (one warp per query row and head).
#include "common.cuh"

namespace {

constexpr int kBM = 128;
constexpr int kBN = 128;
constexpr int kD = 128;
constexpr int kKStages = 3;
constexpr int kVStages = 2;
constexpr int kSBufs = 3;                              // S/P buffers in TMEM
constexpr int kBiasStages = 4;                         // per-key bias ring (beside the K ring)
constexpr int kMaxItems = 128;                         // query tiles one CTA walks, at most
constexpr int kMaxWalkBatch = 256;                     // sequences a walking grid handles
constexpr int kMaxWalkTiles = 2048;                    // query tiles per sequence, likewise
constexpr int kSoftmaxWarps = 8;
constexpr int kThreads = 128 + kSoftmaxWarps * 32;    // warps 0-3 roles, 4-11 softmax
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kStagePitch = 144;   // bytes per staged 64-column row (padded: no bank conflicts)
constexpr float kRescaleThreshold = 8.0f;   // log2 units: move the max only if it grows by > 2^8

// 2^f on [-1/2, 1/2], degree-3 minimax in relative error (7.5e-5), fitted by a
// Remez exchange on the relative error (equi-oscillating error at 5 points).
constexpr float kExp2C0 = 0.9999280571937561f;
constexpr float kExp2C1 = 0.6932609677314758f;
constexpr float kExp2C2 = 0.2426111251115799f;
constexpr float kExp2C3 = 0.0551716685295105f;

struct AttnSmem {
  uint8_t q[2][kBM * 64 * 2];               // Q tile as two 64-column halves (16 KB each)
  uint8_t k[kKStages][2][kBN * 64 * 2];
  uint8_t v[kVStages][2][kBN * 64 * 2];
  float bias[kBiasStages][kBN];
  uint8_t ostage[kSoftmaxWarps][16][kStagePitch];   // epilogue: each warp's 16 rows of O, bf16
  uint64_t q_full;
  uint64_t q_empty;
  uint64_t k_full[kKStages];
  uint64_t k_empty[kKStages];
  uint64_t b_full[kBiasStages];
  uint64_t b_empty[kBiasStages];
  uint64_t v_full[kVStages];
  uint64_t v_empty[kVStages];
  uint64_t s_full[kSBufs];
  uint64_t p_full[kSBufs];                  // P_g stored by every softmax warp, on p_full[g % kSBufs]
  uint64_t o_done[kSBufs];                  // PV_g complete, on o_done[g % kSBufs]
  uint64_t o_free;                          // the epilogue has read O (next query tile may overwrite)
  int4 item[kMaxItems];                     // the CTA's query tiles: (head, tile, seq0, len)
  int2 seq[kMaxWalkBatch];                  // walking grid: each sequence's (first row, length)
  int above[kMaxWalkTiles + 1];             // walking grid: items with a tile above t, at t + 1
  int n_items;
  uint32_t tmem_base;
  int abort_flag;
};

// TMEM columns: S/P buffers at 0, 128 and 256, O at 384 (512 allocated).
constexpr uint32_t kColS0 = 0, kColO = 384, kTmemCols = 512;

__device__ __forceinline__ bool all_alive(bool a) { return __all_sync(0xFFFFFFFFu, a); }

// packed pair arithmetic (one instruction for two fp32 lanes)
__device__ __forceinline__ void ffma2(float& d0, float& d1, float a0, float a1, float b0, float b1,
                                      float c0, float c1) {
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}
__device__ __forceinline__ void fadd2(float& d0, float& d1, float a0, float a1, float b0,
                                      float b1) {
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
__device__ __forceinline__ void fsub2(float& d0, float& d1, float a0, float a1, float b0,
                                      float b1) {
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "sub.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
// exp2 on the FMA pipe, two lanes at once (packed f32x2 additions and FMAs):
// n = rint(x) via the 1.5*2^23 shift, 2^f by the polynomial, 2^n added to the
// exponent field as t << 23 (t = x + 1.5*2^23 holds n in its low mantissa bits;
// the shift's own bits, 0x4B400000, have nine zero low bits and vanish modulo
// 2^32). Inputs below -125 return ~2^-125 (P is bf16; such a weight is zero for
// every purpose here); inputs are <= 8 by construction.
__device__ __forceinline__ void exp2_fma2(float& y0, float& y1, float x0, float x1) {
  x0 = fmaxf(x0, -125.0f);
  x1 = fmaxf(x1, -125.0f);
  float t0, t1, n0, n1, f0, f1, p0, p1;
  fadd2(t0, t1, x0, x1, 12582912.0f, 12582912.0f);
  fsub2(n0, n1, t0, t1, 12582912.0f, 12582912.0f);
  fsub2(f0, f1, x0, x1, n0, n1);
  ffma2(p0, p1, kExp2C3, kExp2C3, f0, f1, kExp2C2, kExp2C2);
  ffma2(p0, p1, p0, p1, f0, f1, kExp2C1, kExp2C1);
  ffma2(p0, p1, p0, p1, f0, f1, kExp2C0, kExp2C0);
  y0 = __uint_as_float(__float_as_uint(p0) + (__float_as_uint(t0) << 23));
  y1 = __uint_as_float(__float_as_uint(p1) + (__float_as_uint(t1) << 23));
}
// acc += the low (lo) or high (hi) bf16 half of a packed pair, widened exactly
// (one mixed-precision add; the same value and rounding as an fp32 add)
__device__ __forceinline__ void add_bf16_lo(float& acc, uint32_t u) {
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\tadd.rn.f32.bf16 %0, l, %0;\n\t}"
      : "+f"(acc)
      : "r"(u));
}
__device__ __forceinline__ void add_bf16_hi(float& acc, uint32_t u) {
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %1;\n\tadd.rn.f32.bf16 %0, h, %0;\n\t}"
      : "+f"(acc)
      : "r"(u));
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

}  // namespace

namespace {

__global__ void __launch_bounds__(kThreads, 1)
    gated_attn_bf16_kernel(const __grid_constant__ CUtensorMap tm_q,
                           const __grid_constant__ CUtensorMap tm_k,
                           const __grid_constant__ CUtensorMap tm_v,
                           const float* __restrict__ s_kept, const float* __restrict__ gain,
                           const float* __restrict__ tau, const int32_t* __restrict__ cu_kept,
                           int total, int max_kept, int n_hq, int n_hkv, int batch,
                           int n_qt, int walk, __nv_bfloat16* __restrict__ out,
                           float* __restrict__ lse, int* status) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (tg::smem_u32(smem_raw) & 1023u)) & 1023u;
  AttnSmem& S = *reinterpret_cast<AttnSmem*>(smem_raw + pad);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    tg::mbar_init(&S.q_full, 1);
    tg::mbar_init(&S.q_empty, 1);
    for (int s = 0; s < kKStages; ++s) {
      tg::mbar_init(&S.k_full[s], 1);    // expect_tx arrival
      tg::mbar_init(&S.k_empty[s], 1);   // S_j computed
    }
    for (int s = 0; s < kBiasStages; ++s) {
      tg::mbar_init(&S.b_full[s], 32);              // every lane of the staging warp
      tg::mbar_init(&S.b_empty[s], kSoftmaxWarps);  // read by every softmax warp
    }
    for (int s = 0; s < kVStages; ++s) {
      tg::mbar_init(&S.v_full[s], 1);
      tg::mbar_init(&S.v_empty[s], 1);
    }
    for (int s = 0; s < kSBufs; ++s) tg::mbar_init(&S.s_full[s], 1);
    for (int s = 0; s < kSBufs; ++s) tg::mbar_init(&S.p_full[s], kSoftmaxWarps);
    for (int s = 0; s < kSBufs; ++s) tg::mbar_init(&S.o_done[s], 1);
    tg::mbar_init(&S.o_free, kSoftmaxWarps);
    S.abort_flag = 0;
    tg::fence_barrier_init();
  }
  if (warp == 2) {
    tg::tmem_alloc(&S.tmem_base, kTmemCols);
    tg::tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tg::tma_prefetch_desc(&tm_q);
    tg::tma_prefetch_desc(&tm_k);
  }
  if (warp == 3 && lane == 0) tg::tma_prefetch_desc(&tm_v);
  tg::tc_fence_before();
  __syncthreads();
  tg::tc_fence_after();
  const uint32_t tmem = S.tmem_base;
  tg::pdl_launch_dependents();
  tg::pdl_wait();   // global memory only from here on

  // The CTA's query tiles, in the order every role walks them. The items (tile,
  // sequence, head) that exist are numbered longest tile first: tile n_qt-1 of every
  // sequence long enough for it and every head, then the next tile down. walk != 0:
  // item v goes to CTA c for v = c, 2G-1-c, 2G+c, ... (a snake, so that long and
  // short items pair up and every CTA's list sums to about the same number of key
  // tiles); thread r finds the CTA's r-th item from the per-sequence tile counts (a
  // binary search over the items-above-tile counts, then the sequence). walk == 0:
  // CTA c takes item c of the numbering over all (tile, sequence, head), skipped when
  // the tile lies beyond its sequence. A sequence whose kept range lies outside
  // [0, total] or is longer than max_kept (n_qt covers max_kept rows) is not
  // attended: it is recorded and gets no tile.
  auto seq_geom = [&](int b) -> int2 {
    const int seq0 = cu_kept[b];
    const int seq1 = cu_kept[b + 1];
    const bool bad = seq0 < 0 || seq1 < seq0 || seq1 > total || seq1 - seq0 > max_kept;
    if (bad) tg::set_status(status, TG_ERR_DEVICE_CHECK);
    return make_int2(seq0, bad ? 0 : seq1 - seq0);
  };
  if (walk && batch == 1) {   // one sequence: item v is tile n_t-1-v/n_hq of head v%n_hq
    if (tid == 0) {
      const int2 g = seq_geom(0);
      const int64_t V = static_cast<int64_t>((g.y + kBM - 1) / kBM) * n_hq;
      const int64_t G = gridDim.x;
      int n = 0;
      for (int64_t r = 0; n < kMaxItems; ++r) {
        const int64_t v = r * G + ((r & 1) ? G - 1 - blockIdx.x : blockIdx.x);
        if (v >= V) break;
        S.item[n++] = make_int4(static_cast<int>(v % n_hq),
                                static_cast<int>(V / n_hq - 1 - v / n_hq), g.x, g.y);
      }
      S.n_items = n;
    }
  } else if (walk) {
    for (int b = tid; b < batch; b += kThreads) S.seq[b] = seq_geom(b);
    __syncthreads();
    for (int t = tid - 1; t < n_qt; t += kThreads) {
      int c = 0;
      for (int b = 0; b < batch; ++b) {
        const int nt = (S.seq[b].y + kBM - 1) / kBM;
        c += nt - 1 - t > 0 ? nt - 1 - t : 0;
      }
      S.above[t + 1] = c * n_hq;
    }
    __syncthreads();
    int found = 0;
    if (tid < kMaxItems) {
      const int64_t G = gridDim.x;
      const int64_t v = tid * G + ((tid & 1) ? G - 1 - blockIdx.x : blockIdx.x);
      if (v < S.above[0]) {
        int lo = 0, hi = n_qt - 1;   // the first tile t with at most v items above it
        while (lo < hi) {
          const int mid = (lo + hi) >> 1;
          if (S.above[mid + 1] <= v) hi = mid; else lo = mid + 1;
        }
        const int k = static_cast<int>(v) - S.above[lo + 1];   // index within tile lo's items
        const int j = k / n_hq;                               // the j-th sequence long enough
        int b = 0;
        for (int seen = 0; b < batch; ++b) {
          if (S.seq[b].y > lo * kBM) {
            if (seen == j) break;
            ++seen;
          }
        }
        S.item[tid] = make_int4(k % n_hq, lo, S.seq[b].x, S.seq[b].y);
        found = 1;
      }
    }
    // a CTA's items are v = c, 2G-1-c, ... in increasing order: the first r past the
    // last item ends the list
    const int n = __syncthreads_count(found);
    if (tid == 0) S.n_items = n;
  } else if (tid == 0) {
    const int64_t i = blockIdx.x;
    const int hq = static_cast<int>(i % n_hq);
    const int b = static_cast<int>((i / n_hq) % batch);
    const int t = n_qt - 1 - static_cast<int>(i / (static_cast<int64_t>(n_hq) * batch));
    const int2 g = seq_geom(b);
    S.n_items = t * kBM < g.y ? 1 : 0;
    S.item[0] = make_int4(hq, t, g.x, g.y);
  }
  __syncthreads();
  const int nq = S.n_items;
  if (nq == 0) {   // uniform: no query tile here
    if (warp == 2) tg::tmem_dealloc(tmem, kTmemCols);
    return;
  }

  if (warp == 0) {
    // ---------------- TMA producer: Q and K tiles ----------------
    if (lane == 0) {
      int g = 0, q_issued = 0;
      bool go = true;
      for (int qi = 0; qi < nq && go; ++qi) {
        const int4 itm = S.item[qi];
        const int hq = itm.x, t = itm.y, seq0 = itm.z, kvh = hq / (n_hq / n_hkv);
        if (qi > 0 && !tg::mbar_wait(&S.q_empty, (qi - 1) & 1, status, &S.abort_flag)) break;
        tg::mbar_arrive_expect_tx(&S.q_full, kBM * kD * 2);
        tg::tma_load_3d(S.q[0], &tm_q, &S.q_full, 0, hq, seq0 + t * kBM);
        tg::tma_load_3d(S.q[1], &tm_q, &S.q_full, 64, hq, seq0 + t * kBM);
        ++q_issued;
        for (int j = 0; j <= t; ++j, ++g) {
          const int s = g % kKStages;
          if (g >= kKStages &&
              !tg::mbar_wait(&S.k_empty[s], ((g / kKStages) - 1) & 1, status, &S.abort_flag)) {
            go = false;
            break;
          }
          tg::mbar_arrive_expect_tx(&S.k_full[s], kBN * kD * 2);
          const int r0 = seq0 + j * kBN;
          tg::tma_load_3d(S.k[s][0], &tm_k, &S.k_full[s], 0, kvh, r0);
          tg::tma_load_3d(S.k[s][1], &tm_k, &S.k_full[s], 64, kvh, r0);
        }
      }
      if (S.abort_flag) {   // let copies in flight land before the CTA exits
        if (q_issued > 0) tg::mbar_wait(&S.q_full, (q_issued - 1) & 1, status, nullptr);
        for (int j = g > kKStages ? g - kKStages : 0; j < g; ++j)
          tg::mbar_wait(&S.k_full[j % kKStages], (j / kKStages) & 1, status, nullptr);
      }
    }
    __syncwarp();
  } else if (warp == 2) {
    // ---------------- bias staging (32 arrivals per K stage) ----------------
    // A register ring keeps the loads of the next kKStages tiles in flight, so the
    // staging keeps pace with the K ring instead of waiting one load per tile.
    // A lookahead cursor walks (query tile, key tile) in the K ring's order.
    int la_q = 0, la_j = 0, n_tiles = 0;
    for (int q = 0; q < nq; ++q) n_tiles += S.item[q].y + 1;
    auto load_next = [&](float* v) {   // the scaled bias of the tile under the cursor
      if (la_q < nq) {
        const int4 itm = S.item[la_q];
        const float gl2 = gain[itm.x] * kLog2e;
#pragma unroll
        for (int u = 0; u < kBN / 32; ++u) {
          const int kp = la_j * kBN + lane + 32 * u;
          v[u] = kp < itm.w && tg::in_bounds(itm.z + kp, total, status) ? gl2 * s_kept[itm.z + kp]
                                                                        : 0.f;
        }
        if (++la_j > itm.y) {
          la_j = 0;
          ++la_q;
        }
      } else {
#pragma unroll
        for (int u = 0; u < kBN / 32; ++u) v[u] = 0.f;
      }
    };
    float v0[kBN / 32], v1[kBN / 32], v2[kBN / 32];
    load_next(v0);
    load_next(v1);
    load_next(v2);
    for (int g = 0; g < n_tiles; ++g) {
      const int s = g % kBiasStages;
      if (g >= kBiasStages &&
          !all_alive(tg::mbar_wait(&S.b_empty[s], ((g / kBiasStages) - 1) & 1, status,
                                   &S.abort_flag)))
        break;
#pragma unroll
      for (int u = 0; u < kBN / 32; ++u) S.bias[s][lane + 32 * u] = v0[u];
      tg::mbar_arrive(&S.b_full[s]);
#pragma unroll
      for (int u = 0; u < kBN / 32; ++u) {
        v0[u] = v1[u];
        v1[u] = v2[u];
      }
      load_next(v2);
    }
  } else if (warp == 3) {
    // ---------------- TMA producer: V tiles ----------------
    if (lane == 0) {
      int g = 0;
      bool go = true;
      for (int qi = 0; qi < nq && go; ++qi) {
        const int4 itm = S.item[qi];
        const int seq0 = itm.z, kvh = itm.x / (n_hq / n_hkv);
        for (int j = 0; j <= itm.y; ++j, ++g) {
          const int s = g % kVStages;
          if (g >= kVStages &&
              !tg::mbar_wait(&S.v_empty[s], ((g / kVStages) - 1) & 1, status, &S.abort_flag)) {
            go = false;
            break;
          }
          tg::mbar_arrive_expect_tx(&S.v_full[s], kBN * kD * 2);
          const int r0 = seq0 + j * kBN;
          tg::tma_load_3d(S.v[s][0], &tm_v, &S.v_full[s], 0, kvh, r0);
          tg::tma_load_3d(S.v[s][1], &tm_v, &S.v_full[s], 64, kvh, r0);
        }
      }
      if (S.abort_flag) {
        for (int j = g > kVStages ? g - kVStages : 0; j < g; ++j)
          tg::mbar_wait(&S.v_full[j % kVStages], (j / kVStages) & 1, status, nullptr);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer: S_0, S_1, S_2, PV_0, S_3, PV_1, ... ----------------
    if (lane == 0) {
      constexpr uint32_t idesc_s = tg::idesc_bf16_f32(kBM, kBN, false, false);
      constexpr uint32_t idesc_o = tg::idesc_bf16_f32(kBM, kD, false, true);
      const uint32_t q0 = tg::smem_u32(S.q[0]);
      auto issue_s = [&](int g) -> bool {
        const int s = g % kKStages;
        if (!tg::mbar_wait(&S.k_full[s], (g / kKStages) & 1, status, &S.abort_flag)) return false;
        tg::tc_fence_after();
        const uint32_t k0 = tg::smem_u32(S.k[s][0]);
        const uint32_t d_s = tmem + kColS0 + 128u * (g % kSBufs);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (kBM * 64 * 2) + (kk & 3) * 32;
          tg::mma_bf16_ss(d_s, tg::smem_desc_sw128(q0 + off, 16, 1024),
                          tg::smem_desc_sw128(k0 + off, 16, 1024), idesc_s, kk != 0);
        }
        tg::mma_commit(&S.s_full[g % kSBufs]);
        tg::mma_commit(&S.k_empty[s]);
        return true;
      };
      bool alive = true;
      int g0 = 0;
      for (int qi = 0; qi < nq && alive; ++qi) {
        const int nt = S.item[qi].y + 1;
        alive = tg::mbar_wait(&S.q_full, qi & 1, status, &S.abort_flag);
        for (int j = 0; j < kSBufs && j < nt && alive; ++j) alive = issue_s(g0 + j);
        if (alive && nt <= kSBufs) tg::mma_commit(&S.q_empty);   // every S of the tile issued
        for (int j = 0; j < nt && alive; ++j) {
          const int g = g0 + j;
          if (!tg::mbar_wait(&S.p_full[g % kSBufs], (g / kSBufs) & 1, status, &S.abort_flag)) {
            alive = false;
            break;
          }
          const int s = g % kVStages;
          if (!tg::mbar_wait(&S.v_full[s], (g / kVStages) & 1, status, &S.abort_flag)) {
            alive = false;
            break;
          }
          if (j == 0 && qi > 0 &&
              !tg::mbar_wait(&S.o_free, (qi - 1) & 1, status, &S.abort_flag)) {
            alive = false;
            break;
          }
          tg::tc_fence_after();
          const uint32_t v0 = tg::smem_u32(S.v[s][0]);
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk) {
            // A = P_g in TMEM (16 keys = 8 packed columns per K step); B = V rows
            // 16kk..16kk+15, MN-major: the two 64-wide dh halves are 16 KB apart
            // (LBO), 8-key groups 1024 B apart (SBO)
            const uint64_t bdesc = tg::smem_desc_sw128(v0 + kk * 16 * 128, kBN * 64 * 2, 1024);
            tg::mma_bf16_ts(tmem + kColO, tmem + kColS0 + 128u * (g % kSBufs) + kk * 8, bdesc,
                            idesc_o, (j | kk) != 0);
          }
          tg::mma_commit(&S.o_done[g % kSBufs]);
          tg::mma_commit(&S.v_empty[s]);
          // S_{g+3} goes into the buffer that held P_g (PV_g is ahead of it in the pipe)
          if (j + kSBufs < nt) {
            if (!issue_s(g + kSBufs)) { alive = false; break; }
            if (j + kSBufs + 1 == nt) tg::mma_commit(&S.q_empty);   // every S of the tile issued
          }
        }
        g0 += nt;
      }
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ---------------- softmax: one warp per 16 query rows ----------------
    // Warp w reaches TMEM lanes 32(w%4)..+31 and the two warps of a lane quarter
    // take its two 16-lane halves. In the 16x256b shape thread l holds rows
    // ra = l/4 and rb = l/4 + 8 of its half at columns 8i + 2(l%4) + {0,1}, i < 16:
    // a row's 128 keys sit in one quad, so its max and sum are two shuffles.
    const int quarter = warp & 3;
    const int half = (warp - 4) >> 2;
    const int row0 = quarter * 32 + half * 16;
    const int ra = row0 + (lane >> 2), rb = ra + 8;   // rows within the tile == TMEM lanes
    const int cq = 2 * (lane & 3);                    // first column within each group of 8
    const uint32_t lane_base = static_cast<uint32_t>(row0) << 16;
    bool alive = true;
    int g0 = 0;
    for (int qi = 0; qi < nq && alive; ++qi) {
      const int4 itm = S.item[qi];
      const int hq = itm.x, t = itm.y, seq0 = itm.z, len = itm.w;
      const float c_h = kLog2e / (sqrtf(static_cast<float>(kD)) * tau[hq]);
      const int nt = t + 1;
      float ma = -INFINITY, mb = -INFINITY;   // running maxima of rows ra, rb
      float la = 0.f, lb = 0.f;               // this thread's share of their sums
      for (int j = 0; j < nt; ++j) {
        const int g = g0 + j;
        const int s = g % kBiasStages;
        const uint32_t sbuf = tmem + lane_base + kColS0 + 128u * (g % kSBufs);
        alive = tg::mbar_wait(&S.s_full[g % kSBufs], (g / kSBufs) & 1, status, &S.abort_flag);
        if (alive) alive = tg::mbar_wait(&S.b_full[s], (g / kBiasStages) & 1, status, &S.abort_flag);
        if (!all_alive(alive)) { alive = false; break; }
        tg::tc_fence_after();
        float z[64];
        {
          uint32_t u[64];
          tg::tmem_ld_16x256b_x16(sbuf, u);
          tg::tmem_ld_wait();
          const float* bias = S.bias[s] + cq;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float2 bb = *reinterpret_cast<const float2*>(bias + 8 * i);
            ffma2(z[4 * i], z[4 * i + 1], __uint_as_float(u[4 * i]), __uint_as_float(u[4 * i + 1]),
                  c_h, c_h, bb.x, bb.y);
            ffma2(z[4 * i + 2], z[4 * i + 3], __uint_as_float(u[4 * i + 2]),
                  __uint_as_float(u[4 * i + 3]), c_h, c_h, bb.x, bb.y);
          }
        }
        __syncwarp();
        if (lane == 0) tg::mbar_arrive(&S.b_empty[s]);   // this warp is done with the bias
        if (j == t) {   // diagonal tile: key column c is visible to row r iff c <= r
#pragma unroll
          for (int i = 0; i < 16; ++i) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int c = 8 * i + cq + e;
              if (c > ra) z[4 * i + e] = -INFINITY;
              if (c > rb) z[4 * i + 2 + e] = -INFINITY;
            }
          }
        }
        float a0 = fmaxf(z[0], z[1]), a1 = fmaxf(z[4], z[5]);
        float b0 = fmaxf(z[2], z[3]), b1 = fmaxf(z[6], z[7]);
#pragma unroll
        for (int i = 2; i < 16; i += 2) {
          a0 = fmax3(a0, z[4 * i], z[4 * i + 1]);
          a1 = fmax3(a1, z[4 * i + 4], z[4 * i + 5]);
          b0 = fmax3(b0, z[4 * i + 2], z[4 * i + 3]);
          b1 = fmax3(b1, z[4 * i + 6], z[4 * i + 7]);
        }
        float mta = fmaxf(a0, a1), mtb = fmaxf(b0, b1);
        mta = fmaxf(mta, __shfl_xor_sync(0xFFFFFFFFu, mta, 1));
        mtb = fmaxf(mtb, __shfl_xor_sync(0xFFFFFFFFu, mtb, 1));
        mta = fmaxf(mta, __shfl_xor_sync(0xFFFFFFFFu, mta, 2));
        mtb = fmaxf(mtb, __shfl_xor_sync(0xFFFFFFFFu, mtb, 2));
        // the running max of a row moves only when the tile max exceeds it by > 2^8
        float alpha_a = 1.f, alpha_b = 1.f;
        bool rescale = false;
        if (j == 0) {
          ma = mta;
          mb = mtb;
        } else {
          if (mta > ma + kRescaleThreshold) {
            alpha_a = tg::exp2_approx(ma - mta);
            ma = mta;
            rescale = true;
          }
          if (mtb > mb + kRescaleThreshold) {
            alpha_b = tg::exp2_approx(mb - mtb);
            mb = mtb;
            rescale = true;
          }
        }
        uint32_t pk[32];
        float sa[2] = {0.f, 0.f}, sb[2] = {0.f, 0.f};
        const float nma = -ma, nmb = -mb;
#pragma unroll
        for (int i = 0; i < 16; i += 2) {
          float x[8];
          fadd2(x[0], x[1], z[4 * i], z[4 * i + 1], nma, nma);
          fadd2(x[2], x[3], z[4 * i + 2], z[4 * i + 3], nmb, nmb);
          fadd2(x[4], x[5], z[4 * i + 4], z[4 * i + 5], nma, nma);
          fadd2(x[6], x[7], z[4 * i + 6], z[4 * i + 7], nmb, nmb);
          float q0, q4;
          exp2_fma2(q0, q4, x[0], x[4]);   // one key in four on the FMA pipe, two at a time
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int ii = i + h;
            const float p0 = h == 0 ? q0 : q4;
            const float p1 = tg::exp2_approx(x[4 * h + 1]);
            const float p2 = tg::exp2_approx(x[4 * h + 2]);
            const float p3 = tg::exp2_approx(x[4 * h + 3]);
            pk[2 * ii] = tg::pack_bf16x2(p0, p1);       // row ra, packed column 4i + l%4
            pk[2 * ii + 1] = tg::pack_bf16x2(p2, p3);   // row rb, the same column
            // the row sums add the bf16 weights that the PV MMA multiplies: numerator
            // and denominator then carry the same rounding, so a key that dominates
            // its row contributes its v exactly, whatever weight the lagging max left it
            add_bf16_lo(sa[0], pk[2 * ii]);
            add_bf16_hi(sa[1], pk[2 * ii]);
            add_bf16_lo(sb[0], pk[2 * ii + 1]);
            add_bf16_hi(sb[1], pk[2 * ii + 1]);
          }
        }
        la = la * alpha_a + (sa[0] + sa[1]);
        lb = lb * alpha_b + (sb[0] + sb[1]);
        if (__any_sync(0xFFFFFFFFu, rescale)) {
          // O must hold PV_{g-1} before it is scaled
          alive = tg::mbar_wait(&S.o_done[(g - 1) % kSBufs], ((g - 1) / kSBufs) & 1, status,
                                &S.abort_flag);
          if (!all_alive(alive)) { alive = false; break; }
          tg::tc_fence_after();
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {   // O columns 64hh .. 64hh+63 of rows ra, rb
            uint32_t o[32];
            const uint32_t oaddr = tmem + lane_base + kColO + 64u * hh;
            tg::tmem_ld_16x256b_x8(oaddr, o);
            tg::tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              o[4 * i] = __float_as_uint(__uint_as_float(o[4 * i]) * alpha_a);
              o[4 * i + 1] = __float_as_uint(__uint_as_float(o[4 * i + 1]) * alpha_a);
              o[4 * i + 2] = __float_as_uint(__uint_as_float(o[4 * i + 2]) * alpha_b);
              o[4 * i + 3] = __float_as_uint(__uint_as_float(o[4 * i + 3]) * alpha_b);
            }
            tg::tmem_st_16x256b_x8(oaddr, o);
          }
        }
        // P_g over S_g: packed bf16 pairs, 64 columns (every S read of these rows is done)
        tg::tmem_st_16x128b_x16(sbuf, pk);
        tg::tmem_st_wait();
        tg::tc_fence_before();
        __syncwarp();
        if (lane == 0) tg::mbar_arrive(&S.p_full[g % kSBufs]);
      }
      if (!alive) break;
      // ---------------- epilogue of this query tile: O / l -> bf16 ----------------
      la += __shfl_xor_sync(0xFFFFFFFFu, la, 1);
      lb += __shfl_xor_sync(0xFFFFFFFFu, lb, 1);
      la += __shfl_xor_sync(0xFFFFFFFFu, la, 2);
      lb += __shfl_xor_sync(0xFFFFFFFFu, lb, 2);
      const int g_last = g0 + nt - 1;
      alive = tg::mbar_wait(&S.o_done[g_last % kSBufs], (g_last / kSBufs) & 1, status,
                            &S.abort_flag);
      if (!all_alive(alive)) { alive = false; break; }
      tg::tc_fence_after();
      uint32_t o[64];
      tg::tmem_ld_16x256b_x16(tmem + lane_base + kColO, o);
      tg::tmem_ld_wait();
      tg::tc_fence_before();
      __syncwarp();
      if (lane == 0) tg::mbar_arrive(&S.o_free);   // O may now be overwritten
      const float ia = 1.f / la, ib = 1.f / lb;
      const int ga = t * kBM + ra, gb = t * kBM + rb;
      if (lse && cq == 0) {   // log-sum-exp of each row's logits (natural log), [n_hq, total]
        constexpr float kLn2 = 0.69314718055994531f;
        if (ga < len && tg::in_bounds(seq0 + ga, total, status))
          lse[static_cast<int64_t>(hq) * total + seq0 + ga] = (ma + __log2f(la)) * kLn2;
        if (gb < len && tg::in_bounds(seq0 + gb, total, status))
          lse[static_cast<int64_t>(hq) * total + seq0 + gb] = (mb + __log2f(lb)) * kLn2;
      }
      // O / l through this warp's staging rows, 64 columns at a time: the quad
      // layout's 4-byte pieces go to shared memory (padded rows, no bank conflicts
      // either way), and each store to global memory writes four whole 128-byte row
      // segments (32 full lines per warp instead of 256 partial sectors)
      uint8_t* stg = &S.ostage[warp - 4][0][0];
      const int qr = lane >> 2;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int ii = 8 * hh + i;
          *reinterpret_cast<uint32_t*>(stg + qr * kStagePitch + (8 * i + cq) * 2) =
              tg::pack_bf16x2(__uint_as_float(o[4 * ii]) * ia, __uint_as_float(o[4 * ii + 1]) * ia);
          *reinterpret_cast<uint32_t*>(stg + (qr + 8) * kStagePitch + (8 * i + cq) * 2) =
              tg::pack_bf16x2(__uint_as_float(o[4 * ii + 2]) * ib,
                              __uint_as_float(o[4 * ii + 3]) * ib);
        }
        __syncwarp();
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int r = 4 * k + (lane >> 3), cb = (lane & 7) * 16;
          const uint4 val = *reinterpret_cast<const uint4*>(stg + r * kStagePitch + cb);
          const int gr = t * kBM + row0 + r;
          if (gr < len && tg::in_bounds(seq0 + gr, total, status))
            *reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(
                out + (static_cast<int64_t>(seq0 + gr) * n_hq + hq) * kD + 64 * hh) + cb) = val;
        }
        __syncwarp();
      }
      g0 += nt;
    }
  }
  tg::tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tg::tc_fence_after();
    tg::tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

namespace {

// ---------------- exact fp32 path ----------------
constexpr int kF32Warps = 4;

__global__ void __launch_bounds__(kF32Warps * 32)
    gated_attn_f32_kernel(const float* __restrict__ q, const float* __restrict__ k,
                          const float* __restrict__ v, const float* __restrict__ s_kept,
                          const float* __restrict__ gain, const float* __restrict__ tau,
                          const int32_t* __restrict__ cu_kept, int batch, int64_t total,
                          int n_hq, int n_hkv, int dh, float* __restrict__ out,
                          float* __restrict__ lse, int* status) {
  tg::pdl_launch_dependents();
  tg::pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t i = static_cast<int64_t>(blockIdx.x) * kF32Warps + (threadIdx.x >> 5);
  const int hq = blockIdx.y;
  if (i >= total) return;
  int b = 0;
  while (b + 1 < batch && cu_kept[b + 1] <= i) ++b;
  const int64_t j0 = cu_kept[b];
  if (j0 < 0 || j0 > i) {   // row i is not inside sequence b's kept range
    if (lane == 0) tg::set_status(status, TG_ERR_DEVICE_CHECK);
    return;
  }
  const int kvh = hq / (n_hq / n_hkv);
  const float scale = 1.f / (sqrtf(static_cast<float>(dh)) * tau[hq]);
  const float g = gain[hq];
  constexpr int kMaxPerLane = 8;   // dh <= 256
  float qv[kMaxPerLane], acc[kMaxPerLane];
  const float* qi = q + (i * n_hq + hq) * dh;
#pragma unroll
  for (int e = 0; e < kMaxPerLane; ++e) {
    const int c = lane + 32 * e;
    qv[e] = c < dh ? qi[c] : 0.f;
    acc[e] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  for (int64_t j = j0; j <= i; ++j) {
    if (!tg::in_bounds(j, total, status)) break;
    const float* kj = k + (j * n_hkv + kvh) * dh;
    float dot = 0.f;
#pragma unroll
    for (int e = 0; e < kMaxPerLane; ++e) {
      const int c = lane + 32 * e;
      if (c < dh) dot = fmaf(qv[e], kj[c], dot);
    }
    for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xFFFFFFFFu, dot, o);
    const float z = dot * scale + g * s_kept[j];
    const float m_new = fmaxf(m, z);
    const float a = expf(m - m_new);
    const float p = expf(z - m_new);
    l = l * a + p;
    const float* vj = v + (j * n_hkv + kvh) * dh;
#pragma unroll
    for (int e = 0; e < kMaxPerLane; ++e) {
      const int c = lane + 32 * e;
      acc[e] = acc[e] * a + (c < dh ? p * vj[c] : 0.f);
    }
    m = m_new;
  }
  if (lse && lane == 0) lse[static_cast<int64_t>(hq) * total + i] = m + logf(l);
  float* oi = out + (i * n_hq + hq) * dh;
#pragma unroll
  for (int e = 0; e < kMaxPerLane; ++e) {
    const int c = lane + 32 * e;
    if (c < dh) oi[c] = acc[e] / l;
  }
}

tg_status launch_attn_bf16(const void* q, const void* k, const void* v, const float* s_kept,
                           const float* gain, const float* tau, const int32_t* cu_kept, int batch,
                           int64_t total, int max_kept, int n_hq, int n_hkv, void* out,
                           float* lse, cudaStream_t st) {
  int* status = tg::status_word();
  if (!status) return TG_ERR_CUDA;
  CUtensorMap tq, tk, tv;
  const uint64_t dq[3] = {kD, static_cast<uint64_t>(n_hq), static_cast<uint64_t>(total)};
  const uint64_t sq[2] = {kD * 2, static_cast<uint64_t>(n_hq) * kD * 2};
  const uint64_t dk[3] = {kD, static_cast<uint64_t>(n_hkv), static_cast<uint64_t>(total)};
  const uint64_t sk[2] = {kD * 2, static_cast<uint64_t>(n_hkv) * kD * 2};
  const uint32_t box[3] = {64, 1, kBM};
  if (!tg::encode_tmap(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, q, dq, sq, box,
                       CU_TENSOR_MAP_SWIZZLE_128B) ||
      !tg::encode_tmap(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, k, dk, sk, box,
                       CU_TENSOR_MAP_SWIZZLE_128B) ||
      !tg::encode_tmap(&tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, v, dk, sk, box,
                       CU_TENSOR_MAP_SWIZZLE_128B))
    return TG_ERR_CUDA;
  const size_t smem = sizeof(AttnSmem) + 1024;
  if (!tg::ensure_smem(reinterpret_cast<const void*>(gated_attn_bf16_kernel),
                       static_cast<int>(smem)))
    return TG_ERR_CUDA;
  const int n_qt = (max_kept + kBM - 1) / kBM;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return TG_ERR_CUDA;
  // one CTA per SM walking query tiles longest first (more CTAs only when an SM's
  // share would exceed kMaxItems tiles); beyond kMaxWalkBatch sequences or
  // kMaxWalkTiles tiles, one CTA per (tile, sequence, head), longest first
  const int64_t items = static_cast<int64_t>(n_qt) * batch * n_hq;
  const int walk = batch <= kMaxWalkBatch && n_qt <= kMaxWalkTiles ? 1 : 0;
  int64_t ctas = items;
  if (walk) {
    ctas = items < sms ? items : sms;
    if (ctas * kMaxItems < items) ctas = (items + kMaxItems - 1) / kMaxItems;
  }
  if (ctas > INT32_MAX) return TG_ERR_UNSUPPORTED;
  return tg::launch(gated_attn_bf16_kernel, dim3(static_cast<unsigned>(ctas)), dim3(kThreads), smem,
                    st, 0, tq, tk, tv, s_kept, gain, tau, cu_kept, static_cast<int>(total), max_kept,
                    n_hq, n_hkv, batch, n_qt, walk, static_cast<__nv_bfloat16*>(out), lse, status);
}

}  // namespace

extern "C" tg_status tg_gated_attention(const void* q, const void* k, const void* v,
                                        tg_dtype dtype, const float* s_kept, const float* gain,
                                        const float* tau, const int32_t* cu_kept, int batch,
                                        int64_t total_kept, int max_kept, int n_hq, int n_hkv,
                                        int head_dim, void* out, float* lse, tg_stream_t stream) {
  tg::NvtxRange nvtx_range("tg_gated_attention");
  if (batch < 0 || total_kept < 0 || max_kept < 0 || n_hq <= 0 || n_hkv <= 0 || head_dim <= 0)
    return TG_ERR_INVALID_ARG;
  if (batch == 0 || total_kept == 0 || max_kept == 0) return TG_OK;
  if (!q || !k || !v || !s_kept || !gain || !tau || !cu_kept || !out) return TG_ERR_INVALID_ARG;
  if (n_hq % n_hkv != 0) return TG_ERR_INVALID_ARG;
  if (max_kept > total_kept) return TG_ERR_INVALID_ARG;
  if (n_hq > 65535 || batch > 65535) return TG_ERR_UNSUPPORTED;
  if (dtype == TG_BF16) {
    if (head_dim != kD) return TG_ERR_UNSUPPORTED;
    if (total_kept > INT32_MAX - kBM || (max_kept + kBM - 1) / kBM > 65535) return TG_ERR_UNSUPPORTED;
    if (!tg::aligned16(q) || !tg::aligned16(k) || !tg::aligned16(v) || !tg::aligned16(out))
      return TG_ERR_MISALIGNED;
    return launch_attn_bf16(q, k, v, s_kept, gain, tau, cu_kept, batch, total_kept, max_kept, n_hq,
                            n_hkv, out, lse, stream);
  }
  if (dtype == TG_F32) {
    if (head_dim > 256) return TG_ERR_UNSUPPORTED;
    const int64_t blocks = (total_kept + kF32Warps - 1) / kF32Warps;
    if (blocks > INT32_MAX) return TG_ERR_UNSUPPORTED;
    int* status = tg::status_word();
    if (!status) return TG_ERR_CUDA;
    dim3 grid(static_cast<unsigned>(blocks), n_hq);
    return tg::launch(gated_attn_f32_kernel, grid, dim3(kF32Warps * 32), 0, stream, 0,
                      static_cast<const float*>(q), static_cast<const float*>(k),
                      static_cast<const float*>(v), s_kept, gain, tau, cu_kept, batch, total_kept,
                      n_hq, n_hkv, head_dim, static_cast<float*>(out), lse, status);
  }
  return TG_ERR_UNSUPPORTED;
}

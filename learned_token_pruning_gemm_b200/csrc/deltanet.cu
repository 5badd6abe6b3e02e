// tg_gated_delta_rule: the gated delta rule of the hybrid model's Gated DeltaNet
// layers, run over the kept tokens only (MarkTechPost page on TokenGate, section
// "Est-ce que cela fonctionne avec les modèles d'attention hybrides ?" and the
// comparison table: TokenGate also prunes the Gated DeltaNet layers). For each
// sequence and head, a state S in R^{dk x dv} starts at zero and, for the
// sequence's kept tokens t in order,
//     S_t = a_t (I - b_t k_t k_t^T) S_{t-1} + b_t k_t v_t^T,   o_t = S_t^T q_t.
//
// Chunked form. Write the update as S_t = a_t S_{t-1} + k_t u_t^T with
// u_t = b_t (v_t - a_t S_{t-1}^T k_t). Inside a chunk of L <= 64 tokens entered
// with state S_in, and with the decay products P_ti = a_{i+1} ... a_t (i <= t) and
// g_t = a_0 ... a_t, unrolling gives
//     S_t = g_t S_in + sum_{i<=t} P_ti k_i u_i^T,
//     (I + A) U = diag(b) V - diag(b g) K S_in,   A_ti = b_t P_ti k_t.k_i (i < t),
// so with T = (I + A)^{-1}
//     U  = T diag(b) V - T diag(b g) K S_in  =  U~ - W S_in,
//     O  = diag(g) Q S_in + (P o Q K^T) U            (P o: lower triangle, diagonal in),
//     S' = g_{L-1} S_in + K^T diag(P_{L-1,.}) U.
// Everything that does not involve S_in (T, W, U~, the masked Q K^T, g and
// P_{L-1,.}) is independent per chunk: dn_prep_kernel computes it for every
// (chunk, head) in parallel into a workspace record. dn_scan_kernel then walks
// each sequence's chunks in order, per (16 value columns, head, sequence): per
// chunk three small products with the state, on the tensor cores.
//
// Precision. The products run as mma.sync m16n8k16 with bf16 operands and fp32
// accumulation. q, k and v are bf16 already, so products of them are exact; an
// fp32 operand (T, W, the masked Q K^T, U, the state) is split into hi = bf16(x) and
// lo = bf16(x - hi), and x.y is taken as hi.y + lo.y, or hi.hi + hi.lo + lo.hi when
// both sides are split: 16 significant bits per operand, fp32 accumulation.
// (These tiles are 16 to 64 wide and each chunk's three products depend on one
// another through the state, so the warp-level MMA, issued and completed inside the
// warp, fits them better than a TMEM round trip per product.)
#include "common.cuh"

namespace {

constexpr int kDk = 128;
constexpr int kC = 64;         // tokens per chunk
constexpr int kCols = 16;      // value columns per scan CTA
constexpr int kThreads = 128;  // four warps
constexpr int kVBlock = 128;   // value columns per pass of the prep's U~ product

// shared-memory row strides (elements): the eight rows one ldmatrix reads start in
// distinct 16-byte bank groups
constexpr int kLdK = kDk + 8;     // [64][128] bf16 tiles: 272 B rows
constexpr int kLdC = kC + 8;      // [64][64] bf16 tiles: 144 B rows
constexpr int kLdN = kCols + 8;   // [.][16] bf16 tiles: 48 B rows
constexpr int kLdF = kC + 4;      // [64][64] fp32 tiles

// workspace record of one (chunk slot, head), laid out as the scan's shared memory
// wants it (rows padded like the tiles above) so that one bulk copy moves it:
//   wh, wl [64][kLdK] bf16   -W = -T diag(b g) K, split
//   qh, ql [64][kLdC] bf16   P o (Q K^T), split
//   g [64], pl [64] f32      g_t, and P_{L-1,i} (zero past the chunk's end)
// then, per group of 16 value columns, ut [64][16] f32: U~ = T diag(b) V
constexpr uint32_t kRecWl = 64 * kLdK * 2;
constexpr uint32_t kRecQh = 2 * kRecWl;
constexpr uint32_t kRecQl = kRecQh + 64 * kLdC * 2;
constexpr uint32_t kRecG = kRecQl + 64 * kLdC * 2;
constexpr uint32_t kRecPl = kRecG + 64 * 4;
constexpr uint32_t kRecUt = kRecPl + 64 * 4;   // 53760: the part every column group reads
constexpr uint32_t kUtGroup = 64 * kCols * 4;  // one column group's U~
__host__ __device__ inline size_t record_bytes(int dv) {
  return kRecUt + static_cast<size_t>(dv / kCols) * kUtGroup;
}

// ---- small device helpers ----
__device__ __forceinline__ void cp16(void* dst, const void* src, bool ok) {
  // 16 bytes, or 16 zero bytes when !ok (src is not read then)
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(tg::smem_u32(dst)), "l"(src),
               "r"(ok ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// bulk copy global -> shared, completing on the mbarrier (bytes: a multiple of 16)
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(tg::smem_u32(dst)), "l"(src), "r"(bytes), "r"(tg::smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void ldsm(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(tg::smem_u32(p)));
}
__device__ __forceinline__ void ldsm_t(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(tg::smem_u32(p)));
}
// c += a b  (a: 16x16 row-major fragment, b: 16x8 column fragment, fp32 c)
__device__ __forceinline__ void mma(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t as_u32(__nv_bfloat162 v) { return *reinterpret_cast<uint32_t*>(&v); }
// (x0, x1) -> packed bf16 pairs hi = bf16(x), lo = bf16(x - hi); x0 in the low half
__device__ __forceinline__ void split2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
  const float2 hf = __bfloat1622float2(h);
  hi = as_u32(h);
  lo = as_u32(__floats2bfloat162_rn(x0 - hf.x, x1 - hf.y));
}

// Fragments built from fp32 shared-memory tiles (row-major, leading dimension ld),
// each element split into bf16 hi/lo pairs:
//   A (16 x 16 at rows r0, cols c0), each column c scaled by sc[c] when sc is given
__device__ __forceinline__ void frag_a_f32(const float* M, int ld, int r0, int c0, int lane,
                                           const float* sc, uint32_t (&hi)[4], uint32_t (&lo)[4]) {
  const int g = lane >> 2, qd = lane & 3;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int r = r0 + g + 8 * (e & 1), c = c0 + 2 * qd + 8 * (e >> 1);
    float2 x = *reinterpret_cast<const float2*>(M + r * ld + c);
    if (sc) {
      x.x *= sc[c];
      x.y *= sc[c + 1];
    }
    split2(x.x, x.y, hi[e], lo[e]);
  }
}
//   B (16 x 8 at rows k0, cols n0 of a [k][n] tile)
__device__ __forceinline__ void frag_b_f32(const float* M, int ld, int k0, int n0, int lane,
                                           uint32_t (&hi)[2], uint32_t (&lo)[2]) {
  const int g = lane >> 2, qd = lane & 3;
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int kr = k0 + 2 * qd + 8 * e;
    split2(M[kr * ld + n0 + g], M[(kr + 1) * ld + n0 + g], hi[e], lo[e]);
  }
}
// c += a b with both operands split: hi.hi + hi.lo + lo.hi
__device__ __forceinline__ void mma3(float (&c)[4], const uint32_t (&ah)[4], const uint32_t (&al)[4],
                                     const uint32_t (&bh)[2], const uint32_t (&bl)[2]) {
  mma(c, ah, bh[0], bh[1]);
  mma(c, ah, bl[0], bl[1]);
  mma(c, al, bh[0], bh[1]);
}

// Operand addressing (thread `lane` of a warp gives one row address of x4 loads):
//   A fragment of rows r0.., cols c0.. of a row-major tile: row r0 + (lane & 15),
//     col c0 + 8 (lane >> 4)                                          [ldsm]
//   B fragments of two 8-wide n tiles from a [k][n] tile (k rows r0.., n cols c0..):
//     row r0 + (lane & 7) + 8 ((lane >> 3) & 1), col c0 + 8 (lane >> 4)  [ldsm_t]
//     -> (r[0], r[1]) for n tile c0, (r[2], r[3]) for n tile c0 + 8
//   B fragments of two n tiles from an [n][k] tile (n rows r0.., k cols c0..):
//     row r0 + (lane & 7) + 8 (lane >> 4), col c0 + 8 ((lane >> 3) & 1)  [ldsm]
//   A fragment of the transpose of a [k][m] tile (A = X^T; X rows r0.. = k, cols c0.. = m):
//     row r0 + (lane & 7) + 8 (lane >> 4), col c0 + 8 ((lane >> 3) & 1)  [ldsm_t]
// Accumulator element e of n tile j: row (lane >> 2) + 8 (e >> 1), col 8 j + 2 (lane & 3) + (e & 1).

// ---- prep: one CTA per (chunk, head, sequence) ----
// Decay products in the log2 domain: with c_t = log2 a_0 + ... + log2 a_t,
// g_t = 2^c_t and P_ti = 2^(c_t - c_i). T = (I + A)^{-1} by 16 x 16 blocks: the
// four diagonal blocks by forward substitution (one thread per column), then block
// rows 1..3 in order, warp j forming T_rj = -T_rr (sum_{j<=k<r} A_rk T_kj) with
// split-operand MMAs. T diag(b g) and T diag(b) are never stored: the W and U~
// products build their A fragments from T with the column scales applied.
struct PrepSmem {
  __nv_bfloat16 k[kC][kLdK];
  __nv_bfloat16 qv[kC][kLdK];      // q, then a block of up to 128 value columns
  float A[kC][kLdF];               // b_t P_ti k_t.k_i below the diagonal, 0 elsewhere
  float T[kC][kLdF];               // (I + A)^{-1}: diagonal blocks and those below them
  float Y[4][16][16];              // per warp: a block row's partial product
  float cl[kC];                    // c_t
  float g[kC];                     // g_t (0 past the chunk's end)
  float b[kC];                     // b_t (0 past the chunk's end)
  float bg[kC];                    // b_t g_t
};

__global__ void __launch_bounds__(kThreads, 3)
    dn_prep_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                   const __nv_bfloat16* __restrict__ v, const float* __restrict__ alpha,
                   const float* __restrict__ beta, const int32_t* __restrict__ cu, int64_t total,
                   int max_seqlen, int n_heads, int dv, uint8_t* __restrict__ ws, int* status) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  PrepSmem& S = *reinterpret_cast<PrepSmem*>(smem_raw);
  const int c = blockIdx.x, h = blockIdx.y, bq = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  tg::pdl_launch_dependents();
  tg::pdl_wait();
  const int64_t s0 = cu[bq], s1 = cu[bq + 1];
  if (s0 < 0 || s1 < s0 || s1 > total || s1 - s0 > max_seqlen) {   // the scan records it
    return;
  }
  const int64_t n = s1 - s0;
  if (static_cast<int64_t>(c) * kC >= n) return;
  const int L = static_cast<int>(n - static_cast<int64_t>(c) * kC < kC ? n - static_cast<int64_t>(c) * kC : kC);
  const int64_t t0 = s0 + static_cast<int64_t>(c) * kC;
  const int64_t slot = s0 / kC + bq + c;
  uint8_t* rec = ws + (slot * n_heads + h) * record_bytes(dv);

  // ---- stage k and q (rows past the chunk's end are zero); decays and writes ----
  for (int i = tid; i < kC * 16; i += kThreads) {
    const int r = i >> 4, p = i & 15;
    const bool ok = r < L && tg::in_bounds(t0 + r, total, status);
    const int64_t row = (t0 + (ok ? r : 0)) * n_heads + h;
    cp16(&S.k[r][p * 8], k + row * kDk + p * 8, ok);
    cp16(&S.qv[r][p * 8], q + row * kDk + p * 8, ok);
  }
  cp_commit();
  if (warp == 0) {   // c_t: an inclusive scan over the chunk, two tokens per lane
    const int t = 2 * lane;
    const float a0 = t < L ? alpha[(t0 + t) * n_heads + h] : 1.f;
    const float a1 = t + 1 < L ? alpha[(t0 + t + 1) * n_heads + h] : 1.f;
    // a decay of 0 is taken as 1e-30 (its products are then below 1e-30, not 0)
    const float l0 = log2f(fmaxf(a0, 1e-30f)), l1 = log2f(fmaxf(a1, 1e-30f));
    float sum = l0 + l1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float y = __shfl_up_sync(0xFFFFFFFFu, sum, o);
      if (lane >= o) sum += y;
    }
    const float c0 = sum - l1, c1 = sum;
    S.cl[t] = c0;
    S.cl[t + 1] = c1;
    const float g0 = t < L ? exp2f(c0) : 0.f, g1 = t + 1 < L ? exp2f(c1) : 0.f;
    const float b0 = t < L ? beta[(t0 + t) * n_heads + h] : 0.f;
    const float b1 = t + 1 < L ? beta[(t0 + t + 1) * n_heads + h] : 0.f;
    S.g[t] = g0;
    S.g[t + 1] = g1;
    S.b[t] = b0;
    S.b[t + 1] = b1;
    S.bg[t] = b0 * g0;
    S.bg[t + 1] = b1 * g1;
  }
  cp_wait_all();
  __syncthreads();

  // ---- K K^T and Q K^T together (warp w: rows 16w .. 16w+15): A, and P o Q K^T ----
  {
    float ak[8][4], aq[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) ak[j][e] = aq[j][e] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      uint32_t fk[4], fq[4];
      ldsm(fk, &S.k[16 * warp + (lane & 15)][16 * kk + 8 * (lane >> 4)]);
      ldsm(fq, &S.qv[16 * warp + (lane & 15)][16 * kk + 8 * (lane >> 4)]);
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t bb[4];
        ldsm(bb, &S.k[16 * np + (lane & 7) + 8 * (lane >> 4)][16 * kk + 8 * ((lane >> 3) & 1)]);
        mma(ak[2 * np], fk, bb[0], bb[1]);
        mma(ak[2 * np + 1], fk, bb[2], bb[3]);
        mma(aq[2 * np], fq, bb[0], bb[1]);
        mma(aq[2 * np + 1], fq, bb[2], bb[3]);
      }
    }
    __nv_bfloat16* qh = reinterpret_cast<__nv_bfloat16*>(rec + kRecQh);
    __nv_bfloat16* ql = reinterpret_cast<__nv_bfloat16*>(rec + kRecQl);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int r = 16 * warp + (lane >> 2) + 8 * hf;
        const int col = 8 * j + 2 * (lane & 3);
        const float cr = S.cl[r], br = S.b[r];
        const float p0 = col <= r ? tg::exp2_approx(cr - S.cl[col]) : 0.f;
        const float p1 = col + 1 <= r ? tg::exp2_approx(cr - S.cl[col + 1]) : 0.f;
        S.A[r][col] = col < r ? br * p0 * ak[j][2 * hf] : 0.f;
        S.A[r][col + 1] = col + 1 < r ? br * p1 * ak[j][2 * hf + 1] : 0.f;
        uint32_t hi, lo;
        split2(p0 * aq[j][2 * hf], p1 * aq[j][2 * hf + 1], hi, lo);
        *reinterpret_cast<uint32_t*>(qh + r * kLdC + col) = hi;
        *reinterpret_cast<uint32_t*>(ql + r * kLdC + col) = lo;
      }
    }
  }
  __syncthreads();   // A complete; q no longer read

  // ---- the first value block loads into q's place during the solve ----
  const int vb = dv < kVBlock ? dv : kVBlock;
  auto stage_v = [&](int c0, int width) {
    const int pieces = width / 8;
    for (int i = tid; i < kC * pieces; i += kThreads) {
      const int r = i / pieces, p = i % pieces;
      const bool ok = r < L;
      cp16(&S.qv[r][p * 8], v + ((t0 + (ok ? r : 0)) * n_heads + h) * dv + c0 + p * 8, ok);
    }
    cp_commit();
  };
  stage_v(0, vb);

  // ---- diagonal blocks of T: thread 16 d + j solves column j of block d ----
  if (tid < kC) {
    const int o = 16 * (tid >> 4), j = tid & 15;
    float x[16];
#pragma unroll
    for (int t = 0; t < 16; ++t) {
      float s2[2] = {t == j ? 1.f : 0.f, 0.f};
#pragma unroll
      for (int i = 0; i < t; ++i) s2[i & 1] = fmaf(-S.A[o + t][o + i], x[i], s2[i & 1]);
      x[t] = s2[0] + s2[1];
    }
#pragma unroll
    for (int t = 0; t < 16; ++t) S.T[o + t][o + j] = x[t];
  }
  __syncthreads();
  // ---- block rows 1..3: warp j forms T_rj (16 x 16) for j < r ----
#pragma unroll 1
  for (int r = 1; r < 4; ++r) {
    if (warp < r) {
      const int j = warp;
      float y[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      for (int kb = j; kb < r; ++kb) {   // sum_k A_rk T_kj
        uint32_t ah[4], al[4];
        frag_a_f32(&S.A[0][0], kLdF, 16 * r, 16 * kb, lane, nullptr, ah, al);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          uint32_t bh[2], bl[2];
          frag_b_f32(&S.T[0][0], kLdF, 16 * kb, 16 * j + 8 * nt, lane, bh, bl);
          mma3(y[nt], ah, al, bh, bl);
        }
      }
      float* yw = &S.Y[warp][0][0];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf)
          *reinterpret_cast<float2*>(yw + ((lane >> 2) + 8 * hf) * 16 + 8 * nt + 2 * (lane & 3)) =
              make_float2(y[nt][2 * hf], y[nt][2 * hf + 1]);
      __syncwarp();
      float tt[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      uint32_t ah[4], al[4];
      frag_a_f32(&S.T[0][0], kLdF, 16 * r, 16 * r, lane, nullptr, ah, al);   // T_rr
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        uint32_t bh[2], bl[2];
        frag_b_f32(yw, 16, 0, 8 * nt, lane, bh, bl);
        mma3(tt[nt], ah, al, bh, bl);
      }
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf)
          *reinterpret_cast<float2*>(&S.T[16 * r + (lane >> 2) + 8 * hf][16 * j + 8 * nt + 2 * (lane & 3)]) =
              make_float2(-tt[nt][2 * hf], -tt[nt][2 * hf + 1]);
    }
    __syncthreads();
  }

  if (tid < kC) {
    reinterpret_cast<float*>(rec + kRecG)[tid] = S.g[tid];
    reinterpret_cast<float*>(rec + kRecPl)[tid] =
        tid < L ? exp2f(S.cl[L - 1] - S.cl[tid]) : 0.f;
  }
  cp_wait_all();
  __syncthreads();

  // ---- -W = -(T diag(b g)) K: warp w rows 16w.., T lower triangular (k tiles <= w) ----
  {
    float acc[16][4];
#pragma unroll
    for (int jn = 0; jn < 16; ++jn) acc[jn][0] = acc[jn][1] = acc[jn][2] = acc[jn][3] = 0.f;
    for (int kk = 0; kk <= warp; ++kk) {
      uint32_t ah[4], al[4];   // T diag(b g): rows 16w.., cols 16kk..
      frag_a_f32(&S.T[0][0], kLdF, 16 * warp, 16 * kk, lane, S.bg, ah, al);
#pragma unroll
      for (int np = 0; np < 8; ++np) {
        uint32_t bb[4];
        ldsm_t(bb, &S.k[16 * kk + (lane & 7) + 8 * ((lane >> 3) & 1)][16 * np + 8 * (lane >> 4)]);
        mma(acc[2 * np], ah, bb[0], bb[1]);
        mma(acc[2 * np], al, bb[0], bb[1]);
        mma(acc[2 * np + 1], ah, bb[2], bb[3]);
        mma(acc[2 * np + 1], al, bb[2], bb[3]);
      }
    }
    __nv_bfloat16* wh = reinterpret_cast<__nv_bfloat16*>(rec);
    __nv_bfloat16* wl = reinterpret_cast<__nv_bfloat16*>(rec + kRecWl);
#pragma unroll
    for (int jn = 0; jn < 16; ++jn) {
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int r = 16 * warp + (lane >> 2) + 8 * hf;
        const int col = 8 * jn + 2 * (lane & 3);
        uint32_t hi, lo;
        split2(-acc[jn][2 * hf], -acc[jn][2 * hf + 1], hi, lo);
        *reinterpret_cast<uint32_t*>(wh + r * kLdK + col) = hi;
        *reinterpret_cast<uint32_t*>(wl + r * kLdK + col) = lo;
      }
    }
  }

  // ---- U~ = (T diag(b)) V, value columns in blocks of 128 ----
  float* ut = reinterpret_cast<float*>(rec + kRecUt);
  for (int c0 = 0; c0 < dv; c0 += kVBlock) {
    const int width = dv - c0 < kVBlock ? dv - c0 : kVBlock;
    if (c0 > 0) {
      __syncthreads();   // every read of the previous block is done
      stage_v(c0, width);
      cp_wait_all();
      __syncthreads();
    }
    float acc[16][4];
#pragma unroll
    for (int jn = 0; jn < 16; ++jn) acc[jn][0] = acc[jn][1] = acc[jn][2] = acc[jn][3] = 0.f;
    for (int kk = 0; kk <= warp; ++kk) {
      uint32_t ah[4], al[4];   // T diag(b)
      frag_a_f32(&S.T[0][0], kLdF, 16 * warp, 16 * kk, lane, S.b, ah, al);
#pragma unroll
      for (int np = 0; np < 8; ++np) {
        if (16 * np < width) {
          uint32_t bb[4];
          ldsm_t(bb, &S.qv[16 * kk + (lane & 7) + 8 * ((lane >> 3) & 1)][16 * np + 8 * (lane >> 4)]);
          mma(acc[2 * np], ah, bb[0], bb[1]);
          mma(acc[2 * np], al, bb[0], bb[1]);
          mma(acc[2 * np + 1], ah, bb[2], bb[3]);
          mma(acc[2 * np + 1], al, bb[2], bb[3]);
        }
      }
    }
#pragma unroll
    for (int jn = 0; jn < 16; ++jn) {
      if (8 * jn < width) {
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const int r = 16 * warp + (lane >> 2) + 8 * hf;
          const int col = c0 + 8 * jn + 2 * (lane & 3);   // group col / 16, column col % 16
          *reinterpret_cast<float2*>(ut + (static_cast<int64_t>(col / kCols) * kC + r) * kCols + col % kCols) =
              make_float2(acc[jn][2 * hf], acc[jn][2 * hf + 1]);
        }
      }
    }
  }
}

// ---- scan: one CTA per (16 value columns, head, sequence), chunks in order ----
// A chunk's stage arrives on one mbarrier from six copies: the chunk's q and k rows
// as two TMA boxes each (64 rows x 64 dims, 128-byte swizzle), the record's shared
// part (53760 B) and this column group's U~ (4 KB) as two bulk copies. The next
// chunk's copies fly during this chunk.
struct __align__(1024) ScanStage {
  uint8_t q[2][kC * 128];                     // [dims 0-63 | 64-127][row][128 B], swizzled
  uint8_t k[2][kC * 128];
  __nv_bfloat16 wh[kC][kLdK], wl[kC][kLdK];   // from here on, the record's shared part:
  __nv_bfloat16 qh[kC][kLdC], ql[kC][kLdC];   //   -W and P o (Q K^T), split;
  float g[kC], pl[kC];                        //   g and P_{L-1,.}
  float ut[kC][kCols];                        // this CTA's columns of U~
};
static_assert(offsetof(ScanStage, ut) - offsetof(ScanStage, wh) == kRecUt,
              "stage layout mirrors the record");
// byte address of 16-byte chunk (row r, dims c .. c+7) of a swizzled q/k tile
__device__ __forceinline__ const uint8_t* sw128(const uint8_t* tile, int r, int c) {
  return tile + (c >> 6) * (kC * 128) + r * 128 + ((((c >> 3) & 7) ^ (r & 7)) << 4);
}
struct ScanSmem {
  ScanStage st[2];
  float s[kDk][kCols];                             // the state's columns, fp32
  __nv_bfloat16 sh[kDk][kLdN], sl[kDk][kLdN];      // the same, split
  __nv_bfloat16 uh[kC][kLdN], ul[kC][kLdN];        // U, split
  __nv_bfloat16 puh[kC][kLdN], pul[kC][kLdN];      // diag(P_{L-1,.}) U, split
  uint64_t full[2];
  int abort_flag;
};

__global__ void __launch_bounds__(kThreads, 1)
    dn_scan_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const int32_t* __restrict__ cu, int64_t total, int max_seqlen, int n_heads,
                   int dv, const uint8_t* __restrict__ ws, __nv_bfloat16* __restrict__ out,
                   int* status) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const uint32_t pad = (1024u - (tg::smem_u32(smem_raw) & 1023u)) & 1023u;
  ScanSmem& S = *reinterpret_cast<ScanSmem*>(smem_raw + pad);
  const int cg = blockIdx.x, h = blockIdx.y, bq = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c0 = cg * kCols;
  if (tid == 0) {
    tg::mbar_init(&S.full[0], 1);
    tg::mbar_init(&S.full[1], 1);
    S.abort_flag = 0;
    tg::fence_barrier_init();
    tg::tma_prefetch_desc(&tm_q);
    tg::tma_prefetch_desc(&tm_k);
  }
  for (int i = tid; i < kDk * kCols; i += kThreads) {   // S = 0
    const int r = i / kCols, col = i % kCols;
    S.s[r][col] = 0.f;
    S.sh[r][col] = __float2bfloat16_rn(0.f);
    S.sl[r][col] = __float2bfloat16_rn(0.f);
  }
  __syncthreads();
  tg::pdl_launch_dependents();
  tg::pdl_wait();
  const int64_t s0 = cu[bq], s1 = cu[bq + 1];
  if (s0 < 0 || s1 < s0 || s1 > total || s1 - s0 > max_seqlen) {
    if (tid == 0 && cg == 0 && h == 0) tg::set_status(status, TG_ERR_DEVICE_CHECK);
    return;
  }
  const int64_t n = s1 - s0;
  const int nch = static_cast<int>((n + kC - 1) / kC);
  const int64_t slot0 = s0 / kC + bq;
  const size_t rb = record_bytes(dv);
  auto rows_of = [&](int ch) {
    const int64_t left = n - static_cast<int64_t>(ch) * kC;
    return static_cast<int>(left < kC ? left : kC);
  };

  // one thread issues a chunk's six copies after arming the barrier with their bytes
  auto stage = [&](int buf, int ch) {
    ScanStage& T = S.st[buf];
    const uint8_t* rec = ws + ((slot0 + ch) * n_heads + h) * rb;
    const int t0 = static_cast<int>(s0 + static_cast<int64_t>(ch) * kC);
    tg::mbar_arrive_expect_tx(&S.full[buf], 4u * kC * 128u + kRecUt + kUtGroup);
    tg::tma_load_3d(T.q[0], &tm_q, &S.full[buf], 0, h, t0);
    tg::tma_load_3d(T.q[1], &tm_q, &S.full[buf], 64, h, t0);
    tg::tma_load_3d(T.k[0], &tm_k, &S.full[buf], 0, h, t0);
    tg::tma_load_3d(T.k[1], &tm_k, &S.full[buf], 64, h, t0);
    bulk_g2s(&T.wh[0][0], rec, kRecUt, &S.full[buf]);
    bulk_g2s(&T.ut[0][0], rec + kRecUt + static_cast<size_t>(cg) * kUtGroup, kUtGroup, &S.full[buf]);
  };

  if (tid == 0 && nch > 0) stage(0, 0);
  for (int ch = 0; ch < nch; ++ch) {
    const int buf = ch & 1;
    // the other buffer was last read before the previous chunk's last barrier
    if (tid == 0 && ch + 1 < nch) stage(buf ^ 1, ch + 1);
    const bool ok = tg::mbar_wait(&S.full[buf], (ch >> 1) & 1, status, &S.abort_flag);
    if (!__syncthreads_and(ok)) {   // a copy never landed: wait (bounded) for the other stage
      if (tid == 0 && ch + 1 < nch)
        tg::mbar_wait(&S.full[buf ^ 1], ((ch + 1) >> 1) & 1, status, nullptr);
      return;
    }
    ScanStage& T = S.st[buf];
    const int64_t t0 = s0 + static_cast<int64_t>(ch) * kC;
    const int L = rows_of(ch);
    if (L < kC) {   // the last chunk: rows past the end hold the next sequence's rows
      for (int i = tid; i < (kC - L) * 16; i += kThreads) {
        const int r = L + (i >> 4), p = i & 15;   // 16 chunks of 16 B per row (both halves)
        const int off = (p >> 3) * (kC * 128) + r * 128 + (p & 7) * 16;
        *reinterpret_cast<uint4*>(T.q[0] + off) = make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(T.k[0] + off) = make_uint4(0, 0, 0, 0);
      }
      __syncthreads();
    }
    const int ra = 16 * warp + (lane >> 2);   // this thread's accumulator rows ra, ra + 8
    // ---- U = U~ - W S and Q S, one pass over the state's 128 rows ----
    float u[2][4], o[2][4];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        u[j][e] = T.ut[ra + 8 * (e >> 1)][8 * j + 2 * (lane & 3) + (e & 1)];
        o[j][e] = 0.f;
      }
    }
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      uint32_t wh[4], wl[4], qa[4], bh[4], bl[4];
      ldsm(wh, &T.wh[16 * warp + (lane & 15)][16 * kk + 8 * (lane >> 4)]);
      ldsm(wl, &T.wl[16 * warp + (lane & 15)][16 * kk + 8 * (lane >> 4)]);
      ldsm(qa, sw128(T.q[0], 16 * warp + (lane & 15), 16 * kk + 8 * (lane >> 4)));
      ldsm_t(bh, &S.sh[16 * kk + (lane & 7) + 8 * ((lane >> 3) & 1)][8 * (lane >> 4)]);
      ldsm_t(bl, &S.sl[16 * kk + (lane & 7) + 8 * ((lane >> 3) & 1)][8 * (lane >> 4)]);
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        mma(u[j], wh, bh[2 * j], bh[2 * j + 1]);
        mma(u[j], wh, bl[2 * j], bl[2 * j + 1]);
        mma(u[j], wl, bh[2 * j], bh[2 * j + 1]);
        mma(o[j], qa, bh[2 * j], bh[2 * j + 1]);
        mma(o[j], qa, bl[2 * j], bl[2 * j + 1]);
      }
    }
    {
      const float ga = T.g[ra], gb = T.g[ra + 8], pa = T.pl[ra], pb = T.pl[ra + 8];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int col = 8 * j + 2 * (lane & 3);
        uint32_t hi, lo;
        split2(u[j][0], u[j][1], hi, lo);
        *reinterpret_cast<uint32_t*>(&S.uh[ra][col]) = hi;
        *reinterpret_cast<uint32_t*>(&S.ul[ra][col]) = lo;
        split2(u[j][2], u[j][3], hi, lo);
        *reinterpret_cast<uint32_t*>(&S.uh[ra + 8][col]) = hi;
        *reinterpret_cast<uint32_t*>(&S.ul[ra + 8][col]) = lo;
        split2(pa * u[j][0], pa * u[j][1], hi, lo);
        *reinterpret_cast<uint32_t*>(&S.puh[ra][col]) = hi;
        *reinterpret_cast<uint32_t*>(&S.pul[ra][col]) = lo;
        split2(pb * u[j][2], pb * u[j][3], hi, lo);
        *reinterpret_cast<uint32_t*>(&S.puh[ra + 8][col]) = hi;
        *reinterpret_cast<uint32_t*>(&S.pul[ra + 8][col]) = lo;
        o[j][0] *= ga;
        o[j][1] *= ga;
        o[j][2] *= gb;
        o[j][3] *= gb;
      }
    }
    __syncthreads();   // U of every row is in shared memory

    // ---- O = diag(g) Q S + (P o Q K^T) U: k tiles up to the diagonal ----
    for (int kk = 0; kk <= warp; ++kk) {
      uint32_t ah[4], al[4], bh[4], bl[4];
      ldsm(ah, &T.qh[16 * warp + (lane & 15)][16 * kk + 8 * (lane >> 4)]);
      ldsm(al, &T.ql[16 * warp + (lane & 15)][16 * kk + 8 * (lane >> 4)]);
      ldsm_t(bh, &S.uh[16 * kk + (lane & 7) + 8 * ((lane >> 3) & 1)][8 * (lane >> 4)]);
      ldsm_t(bl, &S.ul[16 * kk + (lane & 7) + 8 * ((lane >> 3) & 1)][8 * (lane >> 4)]);
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        mma(o[j], ah, bh[2 * j], bh[2 * j + 1]);
        mma(o[j], ah, bl[2 * j], bl[2 * j + 1]);
        mma(o[j], al, bh[2 * j], bh[2 * j + 1]);
      }
    }
#pragma unroll
    for (int j = 0; j < 2; ++j) {
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int r = ra + 8 * hf;
        if (r < L && tg::in_bounds(t0 + r, total, status)) {
          const int col = c0 + 8 * j + 2 * (lane & 3);
          *reinterpret_cast<__nv_bfloat162*>(out + ((t0 + r) * n_heads + h) * dv + col) =
              __floats2bfloat162_rn(o[j][2 * hf], o[j][2 * hf + 1]);
        }
      }
    }

    // ---- S' = g_{L-1} S + K^T diag(P_{L-1,.}) U: warp w takes state rows 32w .. 32w+31 ----
    float sn[2][2][4];
    {
      const float gl = T.g[L - 1];
#pragma unroll
      for (int m = 0; m < 2; ++m)
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
          for (int e = 0; e < 4; ++e)
            sn[m][j][e] = gl * S.s[32 * warp + 16 * m + (lane >> 2) + 8 * (e >> 1)]
                                  [8 * j + 2 * (lane & 3) + (e & 1)];
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t bh[4], bl[4];
      ldsm_t(bh, &S.puh[16 * kk + (lane & 7) + 8 * ((lane >> 3) & 1)][8 * (lane >> 4)]);
      ldsm_t(bl, &S.pul[16 * kk + (lane & 7) + 8 * ((lane >> 3) & 1)][8 * (lane >> 4)]);
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        uint32_t ka[4];
        ldsm_t(ka, sw128(T.k[0], 16 * kk + (lane & 7) + 8 * (lane >> 4),
                         32 * warp + 16 * m + 8 * ((lane >> 3) & 1)));
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          mma(sn[m][j], ka, bh[2 * j], bh[2 * j + 1]);
          mma(sn[m][j], ka, bl[2 * j], bl[2 * j + 1]);
        }
      }
    }
    __syncthreads();   // every read of the old state and of this stage is done
#pragma unroll
    for (int m = 0; m < 2; ++m) {
#pragma unroll
      for (int j = 0; j < 2; ++j) {
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const int r = 32 * warp + 16 * m + (lane >> 2) + 8 * hf;
          const int col = 8 * j + 2 * (lane & 3);
          const float x0 = sn[m][j][2 * hf], x1 = sn[m][j][2 * hf + 1];
          *reinterpret_cast<float2*>(&S.s[r][col]) = make_float2(x0, x1);
          uint32_t hi, lo;
          split2(x0, x1, hi, lo);
          *reinterpret_cast<uint32_t*>(&S.sh[r][col]) = hi;
          *reinterpret_cast<uint32_t*>(&S.sl[r][col]) = lo;
        }
      }
    }
  }
}

}  // namespace

extern "C" size_t tg_gated_delta_rule_workspace_size(int batch, int64_t total, int n_heads,
                                                     int head_dim_v) {
  if (batch <= 0 || total <= 0 || n_heads <= 0 || head_dim_v <= 0) return 0;
  return static_cast<size_t>(total / kC + batch) * static_cast<size_t>(n_heads) *
         record_bytes(head_dim_v);
}

extern "C" tg_status tg_gated_delta_rule(const void* q, const void* k, const void* v,
                                         tg_dtype dtype, const float* alpha, const float* beta,
                                         const int32_t* cu_seqlens, int batch, int64_t total,
                                         int max_seqlen, int n_heads, int head_dim_k,
                                         int head_dim_v, void* out, void* workspace,
                                         size_t workspace_bytes, tg_stream_t stream) {
  tg::NvtxRange nvtx_range("tg_gated_delta_rule");
  if (batch < 0 || total < 0 || max_seqlen < 0 || n_heads <= 0 || head_dim_k <= 0 || head_dim_v <= 0)
    return TG_ERR_INVALID_ARG;
  if (batch == 0 || total == 0 || max_seqlen == 0) return TG_OK;
  if (!q || !k || !v || !alpha || !beta || !cu_seqlens || !out) return TG_ERR_INVALID_ARG;
  if (dtype != TG_BF16 || head_dim_k != kDk || head_dim_v % kCols != 0 || head_dim_v > 1024)
    return TG_ERR_UNSUPPORTED;
  if (n_heads > 65535 || batch > 65535) return TG_ERR_UNSUPPORTED;
  if (!tg::aligned16(q) || !tg::aligned16(k) || !tg::aligned16(v) || !tg::aligned16(out) ||
      (reinterpret_cast<uintptr_t>(alpha) & 3) || (reinterpret_cast<uintptr_t>(beta) & 3))
    return TG_ERR_MISALIGNED;
  const size_t need = tg_gated_delta_rule_workspace_size(batch, total, n_heads, head_dim_v);
  if (!workspace || workspace_bytes < need) return TG_ERR_WORKSPACE;
  if (!tg::aligned16(workspace)) return TG_ERR_MISALIGNED;
  int* st = tg::status_word();
  if (!st) return TG_ERR_CUDA;
  if (!tg::ensure_smem(reinterpret_cast<const void*>(dn_prep_kernel), static_cast<int>(sizeof(PrepSmem))) ||
      !tg::ensure_smem(reinterpret_cast<const void*>(dn_scan_kernel), static_cast<int>(sizeof(ScanSmem) + 1024)))
    return TG_ERR_CUDA;
  const auto* qb = static_cast<const __nv_bfloat16*>(q);
  const auto* kb = static_cast<const __nv_bfloat16*>(k);
  if (total > INT32_MAX - kC) return TG_ERR_UNSUPPORTED;
  CUtensorMap tq, tk;   // (dims, heads, rows) views, 64 x 1 x 64 boxes, 128-byte swizzle
  const uint64_t dims[3] = {kDk, static_cast<uint64_t>(n_heads), static_cast<uint64_t>(total)};
  const uint64_t strides[2] = {kDk * 2, static_cast<uint64_t>(n_heads) * kDk * 2};
  const uint32_t box[3] = {64, 1, kC};
  if (!tg::encode_tmap(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, q, dims, strides, box,
                       CU_TENSOR_MAP_SWIZZLE_128B) ||
      !tg::encode_tmap(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, k, dims, strides, box,
                       CU_TENSOR_MAP_SWIZZLE_128B))
    return TG_ERR_CUDA;
  const int n_chunks = static_cast<int>((static_cast<int64_t>(max_seqlen) + kC - 1) / kC);
  tg_status r = tg::launch(dn_prep_kernel, dim3(n_chunks, n_heads, batch), dim3(kThreads),
                           sizeof(PrepSmem), stream, 0, qb, kb, static_cast<const __nv_bfloat16*>(v),
                           alpha, beta, cu_seqlens, total, max_seqlen, n_heads, head_dim_v,
                           static_cast<uint8_t*>(workspace), st);
  if (r != TG_OK) return r;
  return tg::launch(dn_scan_kernel, dim3(head_dim_v / kCols, n_heads, batch), dim3(kThreads),
                    sizeof(ScanSmem) + 1024, stream, 0, tq, tk, cu_seqlens, total, max_seqlen, n_heads,
                    head_dim_v, static_cast<const uint8_t*>(workspace),
                    static_cast<__nv_bfloat16*>(out), st);
}

// tg_gated_delta_rule: the gated delta rule of the hybrid model's Gated DeltaNet
// layers, run over the kept tokens only (MarkTechPost page on TokenGate, section
// "Est-ce que cela fonctionne avec les modèles d'attention hybrides ?" and the
// comparison table: TokenGate also prunes the Gated DeltaNet layers). For each
// sequence and head, a state S in R^{dk x dv} starts at zero and, for the
// sequence's kept tokens t in order,
//     S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T,   o_t = S_t^T q_t.
//
// Column c of S evolves on its own: s' = alpha s + beta k (v_c - alpha k.s). So a
// CTA takes 16 value columns of one (head, sequence) and keeps them in registers:
// four adjacent lanes share a column, each holding 32 of its 128 key entries, so
// the two dot products per token (k.s before the update, q.s after it) are a
// partial sum plus two shuffles. The recurrence is sequential in t; what the
// kernel does in parallel is the columns (dv / 16 CTAs per head) and the heads.
// Each CTA stages 32 tokens at a time (k, q, its v columns, alpha, beta) in
// shared memory with cp.async, double-buffered so the next chunk loads while this
// one runs, and writes its outputs 32 tokens at a time.
#include "common.cuh"

namespace {

constexpr int kDk = 128;
constexpr int kCols = 16;           // value columns per CTA
constexpr int kParts = 4;           // lanes per column
constexpr int kPer = kDk / kParts;  // key entries per lane
constexpr int kThreads = kCols * kParts;
constexpr int kChunk = 32;          // tokens staged per buffer

struct DnSmem {
  __nv_bfloat16 k[2][kChunk][kDk];
  __nv_bfloat16 q[2][kChunk][kDk];
  __nv_bfloat16 v[2][kChunk][kCols];
  float a[2][kChunk];
  float b[2][kChunk];
  __nv_bfloat16 o[kChunk][kCols];
};

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(tg::smem_u32(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(tg::smem_u32(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_one() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

__global__ void __launch_bounds__(kThreads)
    gated_delta_rule_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                            const __nv_bfloat16* __restrict__ v, const float* __restrict__ alpha,
                            const float* __restrict__ beta, const int32_t* __restrict__ cu,
                            int64_t total, int n_heads, int dv, __nv_bfloat16* __restrict__ out,
                            int* status) {
  __shared__ __align__(16) DnSmem S;
  const int cg = blockIdx.x, h = blockIdx.y, bq = blockIdx.z;
  const int tid = threadIdx.x;
  const int col = tid / kParts;       // 0..15 (lanes 4c..4c+3 of a warp share a column)
  const int part = tid % kParts;
  tg::pdl_launch_dependents();
  tg::pdl_wait();
  const int64_t t0 = cu[bq], t1 = cu[bq + 1];
  if (t0 < 0 || t1 < t0 || t1 > total) {
    if (tid == 0 && cg == 0 && h == 0) tg::set_status(status, TG_ERR_DEVICE_CHECK);
    return;
  }
  const int64_t n = t1 - t0;
  const int c0 = cg * kCols;

  // stage tokens [tb, tb + kChunk) of the sequence into buffer buf (rows past the
  // end are not loaded; the loop below never reads them)
  auto stage = [&](int buf, int64_t tb) {
    const int rows = static_cast<int>(n - tb < kChunk ? n - tb : kChunk);
    // k and q: rows x 256 B each, 16-byte pieces
    for (int i = tid; i < rows * (kDk / 8); i += kThreads) {
      const int r = i / (kDk / 8), p = i % (kDk / 8);
      const int64_t g = ((t0 + tb + r) * n_heads + h) * kDk + p * 8;
      cp_async16(&S.k[buf][r][p * 8], k + g);
      cp_async16(&S.q[buf][r][p * 8], q + g);
    }
    // v: this CTA's 16 columns = 32 B per row, two 16-byte pieces
    for (int i = tid; i < rows * 2; i += kThreads) {
      const int r = i / 2, p = i % 2;
      cp_async16(&S.v[buf][r][p * 8], v + ((t0 + tb + r) * n_heads + h) * dv + c0 + p * 8);
    }
    for (int i = tid; i < rows; i += kThreads) {
      cp_async4(&S.a[buf][i], alpha + (t0 + tb + i) * n_heads + h);
      cp_async4(&S.b[buf][i], beta + (t0 + tb + i) * n_heads + h);
    }
    cp_async_commit();
  };

  float s[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) s[i] = 0.f;

  if (n > 0) stage(0, 0);
  int buf = 0;
  for (int64_t tb = 0; tb < n; tb += kChunk, buf ^= 1) {
    const int rows = static_cast<int>(n - tb < kChunk ? n - tb : kChunk);
    if (tb + kChunk < n) {
      stage(buf ^ 1, tb + kChunk);   // the next chunk loads while this one runs
      cp_async_wait_one();
    } else {
      cp_async_wait_all();
    }
    __syncthreads();
    for (int r = 0; r < rows; ++r) {
      const uint4* kr = reinterpret_cast<const uint4*>(&S.k[buf][r][part * kPer]);
      const uint4* qr = reinterpret_cast<const uint4*>(&S.q[buf][r][part * kPer]);
      float kf[kPer], qf[kPer];
#pragma unroll
      for (int u = 0; u < kPer / 8; ++u) {
        const uint4 kk = kr[u], qq = qr[u];
        const uint32_t kw[4] = {kk.x, kk.y, kk.z, kk.w}, qw[4] = {qq.x, qq.y, qq.z, qq.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          kf[8 * u + 2 * e] = __uint_as_float(kw[e] << 16);
          kf[8 * u + 2 * e + 1] = __uint_as_float(kw[e] & 0xFFFF0000u);
          qf[8 * u + 2 * e] = __uint_as_float(qw[e] << 16);
          qf[8 * u + 2 * e + 1] = __uint_as_float(qw[e] & 0xFFFF0000u);
        }
      }
      // k.s over this column (four partial sums, then the column's four lanes)
      float d4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int i = 0; i < kPer; ++i) d4[i & 3] = fmaf(kf[i], s[i], d4[i & 3]);
      float dot = (d4[0] + d4[1]) + (d4[2] + d4[3]);
      dot += __shfl_xor_sync(0xFFFFFFFFu, dot, 1);
      dot += __shfl_xor_sync(0xFFFFFFFFu, dot, 2);
      const float a = S.a[buf][r], be = S.b[buf][r];
      const float vc = __bfloat162float(S.v[buf][r][col]);
      const float w = be * (vc - a * dot);
      // s <- a s + w k ; then o = q.s
      float o4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        s[i] = fmaf(a, s[i], w * kf[i]);
        o4[i & 3] = fmaf(qf[i], s[i], o4[i & 3]);
      }
      float o = (o4[0] + o4[1]) + (o4[2] + o4[3]);
      o += __shfl_xor_sync(0xFFFFFFFFu, o, 1);
      o += __shfl_xor_sync(0xFFFFFFFFu, o, 2);
      if (part == 0) S.o[r][col] = __float2bfloat16_rn(o);
    }
    __syncthreads();   // the chunk's outputs are in shared memory; its buffer may be reused
    // rows x 32 B: two 16-byte pieces per token
    for (int i = tid; i < rows * 2; i += kThreads) {
      const int r = i / 2, p = i % 2;
      *reinterpret_cast<uint4*>(out + ((t0 + tb + r) * n_heads + h) * dv + c0 + p * 8) =
          *reinterpret_cast<const uint4*>(&S.o[r][p * 8]);
    }
    __syncthreads();   // S.o is rewritten by the next chunk
  }
}

}  // namespace

extern "C" tg_status tg_gated_delta_rule(const void* q, const void* k, const void* v,
                                         tg_dtype dtype, const float* alpha, const float* beta,
                                         const int32_t* cu_seqlens, int batch, int64_t total,
                                         int n_heads, int head_dim_k, int head_dim_v, void* out,
                                         tg_stream_t stream) {
  tg::NvtxRange nvtx_range("tg_gated_delta_rule");
  if (batch < 0 || total < 0 || n_heads <= 0 || head_dim_k <= 0 || head_dim_v <= 0)
    return TG_ERR_INVALID_ARG;
  if (batch == 0 || total == 0) return TG_OK;
  if (!q || !k || !v || !alpha || !beta || !cu_seqlens || !out) return TG_ERR_INVALID_ARG;
  if (dtype != TG_BF16 || head_dim_k != kDk || head_dim_v % kCols != 0 || head_dim_v > 1024)
    return TG_ERR_UNSUPPORTED;
  if (n_heads > 65535 || batch > 65535) return TG_ERR_UNSUPPORTED;
  if (!tg::aligned16(q) || !tg::aligned16(k) || !tg::aligned16(v) || !tg::aligned16(out) ||
      (reinterpret_cast<uintptr_t>(alpha) & 3) || (reinterpret_cast<uintptr_t>(beta) & 3))
    return TG_ERR_MISALIGNED;
  int* st = tg::status_word();
  if (!st) return TG_ERR_CUDA;
  return tg::launch(gated_delta_rule_kernel, dim3(head_dim_v / kCols, n_heads, batch),
                    dim3(kThreads), 0, stream, 0, static_cast<const __nv_bfloat16*>(q),
                    static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v),
                    alpha, beta, cu_seqlens, total, n_heads, head_dim_v,
                    static_cast<__nv_bfloat16*>(out), st);
}

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
// eight adjacent lanes share a column, each holding 16 of its 128 key entries, so a
// dot product is a partial sum plus three shuffles. After token t's update the
// same state gives both o_t = q_t.s and the next token's k_{t+1}.s, so the two are
// reduced together: one round of shuffles per token on the sequential chain. The
// recurrence is sequential in t; what the kernel does in parallel is the columns
// (dv / 16 CTAs per head) and the heads.
// Each CTA stages 32 tokens at a time (k, q, its v columns, alpha, beta) in
// shared memory with cp.async, double-buffered so the next chunk loads while this
// one runs, and writes its outputs 32 tokens at a time.
#include "common.cuh"

namespace {

constexpr int kDk = 128;
constexpr int kCols = 16;           // value columns per CTA
constexpr int kParts = 8;           // lanes per column
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

  // this lane's 16 entries of a staged bf16 row, widened to fp32
  auto row16 = [&](const __nv_bfloat16* src, float* f) {
    const uint4* p = reinterpret_cast<const uint4*>(src + part * kPer);
#pragma unroll
    for (int u = 0; u < kPer / 8; ++u) {
      const uint4 w4 = p[u];
      const uint32_t w[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        f[8 * u + 2 * e] = __uint_as_float(w[e] << 16);
        f[8 * u + 2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
      }
    }
  };
  auto col_sum = [&](float x) {   // over the column's eight lanes
    x += __shfl_xor_sync(0xFFFFFFFFu, x, 1);
    x += __shfl_xor_sync(0xFFFFFFFFu, x, 2);
    x += __shfl_xor_sync(0xFFFFFFFFu, x, 4);
    return x;
  };

  if (n > 0) stage(0, 0);
  int buf = 0;
  float dot = 0.f;   // k_t . s_{t-1} for the next token (zero state: zero)
  for (int64_t tb = 0; tb < n; tb += kChunk, buf ^= 1) {
    const int rows = static_cast<int>(n - tb < kChunk ? n - tb : kChunk);
    if (tb + kChunk < n) {
      stage(buf ^ 1, tb + kChunk);   // the next chunk loads while this one runs
      cp_async_wait_one();
    } else {
      cp_async_wait_all();
    }
    __syncthreads();
    if (tb > 0) {   // the first token of a chunk: its k.s was not formed with the last output
      float kf[kPer];
      row16(S.k[buf][0], kf);
      float d4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int i = 0; i < kPer; ++i) d4[i & 3] = fmaf(kf[i], s[i], d4[i & 3]);
      dot = col_sum((d4[0] + d4[1]) + (d4[2] + d4[3]));
    }
    for (int r = 0; r < rows; ++r) {
      float kf[kPer], qf[kPer], kn[kPer];
      row16(S.k[buf][r], kf);
      row16(S.q[buf][r], qf);
      const bool has_next = r + 1 < rows;
      if (has_next) row16(S.k[buf][r + 1], kn);
      const float a = S.a[buf][r], be = S.b[buf][r];
      const float vc = __bfloat162float(S.v[buf][r][col]);
      const float w = be * (vc - a * dot);
      // s <- a s + w k; then o_t = q_t . s and the next token's k . s, reduced together
      float o4[4] = {0.f, 0.f, 0.f, 0.f}, n4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        s[i] = fmaf(a, s[i], w * kf[i]);
        o4[i & 3] = fmaf(qf[i], s[i], o4[i & 3]);
        if (has_next) n4[i & 3] = fmaf(kn[i], s[i], n4[i & 3]);
      }
      float o = (o4[0] + o4[1]) + (o4[2] + o4[3]);
      float dn = (n4[0] + n4[1]) + (n4[2] + n4[3]);
#pragma unroll
      for (int off = 1; off < kParts; off <<= 1) {
        o += __shfl_xor_sync(0xFFFFFFFFu, o, off);
        dn += __shfl_xor_sync(0xFFFFFFFFu, dn, off);
      }
      dot = dn;
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

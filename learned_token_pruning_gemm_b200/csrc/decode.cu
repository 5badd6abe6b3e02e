// Decode over the compacted cache (MarkTechPost page on TokenGate, section
// "Comment déployer TokenGate ?": generation runs on the cache that the pruned
// prefill leaves behind, bounded by max_kept_prefill_tokens; section "Qu'est-ce
// que l'attention gérée par des tokens ?": each kept token's score is a logit bias
// with a per-head gain, and a per-head temperature scales the logits).
//
// tg_cache_append: row cache_len[b] of sequence b's cache gets the new token's
// k, v and score; cache_len[b] grows by one.
//
// tg_gated_decode: one new query row per sequence over its cache rows
// j < cache_len[b]:
//     z_j = q . k_j / (sqrt(dh) tau_h) + g_h s_j,   O = sum_j softmax_j(z) v_j.
// The cache is read once, so the work is bound by HBM bandwidth (a GEMV per
// head, no tensor-core shape). It is split along the keys: one CTA per
// (64-key chunk, KV head, sequence) loads the chunk's K and V rows of that KV
// head with two TMA boxes each (64 dims x 64 rows, 128-byte swizzle, 32 KB in
// all) and serves every query head of the GQA group from them: logits in fp32
// (log2 domain), the running max m and sum l of 2^(z - m), and the unnormalised
// sum of 2^(z - m) v. Everything a CTA reads besides the chunk (the cache
// length, the chunk's scores, the group's queries, gains and temperatures) is
// requested at once, and the TMA copy goes out as soon as the length is known.
// Each CTA writes one partial per (sequence, query head, chunk) to a
// caller-provided workspace. A second kernel merges a row's partials in chunk
// order (a fixed order: the result does not depend on timing) and writes
// O = sum_c 2^(m_c - M) o_c / sum_c 2^(m_c - M) l_c in bf16.
// (A CTA walking several chunks through a TMA ring measured slower at every
// batch and length tried, up to 16 sequences of 16k keys: fewer CTAs per SM hold
// fewer bytes in flight.)
#include <mutex>

#include "common.cuh"

namespace {

constexpr int kDh = 128;
constexpr int kChunk = 64;            // keys per split CTA
constexpr int kThreads = 128;
constexpr int kMaxGroup = 8;          // query heads per KV head
constexpr int kPartial = kDh + 2;     // o[dh], m, l (fp32)
constexpr float kLog2e = 1.4426950408889634f;

// Shared memory: this header, then the chunk's 32 KB (K then V, each two
// 64-column halves of 64 rows x 128 B, 128B-swizzled, 1024-byte aligned).
struct DecSmem {
  float q[kMaxGroup][kDh];            // the group's queries, scaled into the log2 domain
  float p[kMaxGroup][kChunk];         // logits, then 2^(z - m)
  uint64_t full;
  int abort_flag;
};
constexpr uint32_t kHalfBytes = kChunk * 64 * 2;                            // 8 KB
constexpr uint32_t kTileBytes = 4 * kHalfBytes;                             // K and V
constexpr uint32_t kHeadBytes = (sizeof(DecSmem) + 1023) / 1024 * 1024;
constexpr size_t kDecodeSmem = 1024 + kHeadBytes + kTileBytes;

// byte offset of element e (0..127) of row j inside a [2][64 rows x 128 B] swizzled tile
__device__ __forceinline__ uint32_t sw_off(int j, int e) {
  const int half = e >> 6, ee = e & 63;
  return half * (kChunk * 128) + j * 128 + ((((ee >> 3) ^ (j & 7)) << 4) | ((ee & 7) << 1));
}

__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

// One CTA per (64-key chunk, KV head, sequence).
__global__ void __launch_bounds__(kThreads)
    decode_split_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                        const __nv_bfloat16* __restrict__ q, const float* __restrict__ s_cache,
                        const int32_t* __restrict__ cache_len, int cap, int max_len, int n_hq,
                        int n_hkv, const float* __restrict__ gain, const float* __restrict__ tau,
                        float* __restrict__ partial, int n_split, int* status) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (tg::smem_u32(smem_raw) & 1023u)) & 1023u;
  DecSmem& S = *reinterpret_cast<DecSmem*>(smem_raw + pad);
  uint8_t* const kt = smem_raw + pad + kHeadBytes;   // K halves, then V halves
  uint8_t* const vt = kt + 2 * kHalfBytes;
  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = n_hq / n_hkv;
  if (tid == 0) {
    tg::mbar_init(&S.full, 1);
    S.abort_flag = 0;
    tg::fence_barrier_init();
    tg::tma_prefetch_desc(&tm_k);
    tg::tma_prefetch_desc(&tm_v);
  }
  __syncthreads();
  tg::pdl_launch_dependents();
  tg::pdl_wait();   // global memory only from here on

  // every independent load at once: the length, key j's score, this thread's
  // query element d = tid of each head of the group, the heads' gains and tau
  const int j0 = split * kChunk;
  const int j = tid & (kChunk - 1);
  const int len = cache_len[b];
  const float sv_raw = j0 + j < cap ? s_cache[static_cast<int64_t>(b) * cap + j0 + j] : 0.f;
  static_assert(kThreads == kDh, "thread d loads query element d");
  float qv[kMaxGroup], cv[kMaxGroup], gv[kMaxGroup / 2];
#pragma unroll
  for (int h = 0; h < kMaxGroup; ++h) {
    const int hq = kvh * G + h;
    qv[h] = h < G ? __bfloat162float(q[(static_cast<int64_t>(b) * n_hq + hq) * kDh + tid]) : 0.f;
    cv[h] = h < G ? tau[hq] : 1.f;
  }
#pragma unroll
  for (int u = 0; u < kMaxGroup / 2; ++u) {
    const int h = (tid >> 6) + 2 * u;
    gv[u] = h < G ? gain[kvh * G + h] * kLog2e : 0.f;
  }
  if (len < 0 || len > cap || len > max_len) return;   // the combine kernel records it
  if (j0 >= len) return;                                // this chunk is past the cache's end
  if (tid == 0) {
    const int row = b * cap + j0;   // token coordinate in the (dh, heads, rows) view
    tg::mbar_arrive_expect_tx(&S.full, kTileBytes);
    tg::tma_load_3d(kt, &tm_k, &S.full, 0, kvh, row);
    tg::tma_load_3d(kt + kHalfBytes, &tm_k, &S.full, 64, kvh, row);
    tg::tma_load_3d(vt, &tm_v, &S.full, 0, kvh, row);
    tg::tma_load_3d(vt + kHalfBytes, &tm_v, &S.full, 64, kvh, row);
  }
#pragma unroll
  for (int h = 0; h < kMaxGroup; ++h)
    if (h < G) S.q[h][tid] = qv[h] * (kLog2e / (sqrtf(static_cast<float>(kDh)) * cv[h]));
  const int nv = min(kChunk, len - j0);   // valid rows of the chunk
  const int e = 2 * (tid & 63);           // this thread's output dims e, e + 1
  float o0[kMaxGroup / 2], o1[kMaxGroup / 2];
#pragma unroll
  for (int u = 0; u < kMaxGroup / 2; ++u) o0[u] = o1[u] = 0.f;
  __syncthreads();
  const bool ok = tg::mbar_wait(&S.full, 0, status, &S.abort_flag);
  if (!__syncthreads_and(ok)) return;   // the copy never landed (recorded in the status)

  // ---- logits: thread t takes key j = t % 64 and heads h = t / 64, t / 64 + 2, ... ----
  {
    float acc[kMaxGroup / 2];
#pragma unroll
    for (int u = 0; u < kMaxGroup / 2; ++u) acc[u] = 0.f;
#pragma unroll 4
    for (int cc = 0; cc < kDh / 8; ++cc) {
      const uint4 kk = *reinterpret_cast<const uint4*>(kt + sw_off(j, 8 * cc));
      const float kf[8] = {bf16_lo(kk.x), bf16_hi(kk.x), bf16_lo(kk.y), bf16_hi(kk.y),
                           bf16_lo(kk.z), bf16_hi(kk.z), bf16_lo(kk.w), bf16_hi(kk.w)};
#pragma unroll
      for (int u = 0; u < kMaxGroup / 2; ++u) {
        const int h = (tid >> 6) + 2 * u;
        if (h < G) {
          const float4 q0 = *reinterpret_cast<const float4*>(&S.q[h][8 * cc]);
          const float4 q1 = *reinterpret_cast<const float4*>(&S.q[h][8 * cc + 4]);
          float a = acc[u];
          a = fmaf(q0.x, kf[0], a); a = fmaf(q0.y, kf[1], a);
          a = fmaf(q0.z, kf[2], a); a = fmaf(q0.w, kf[3], a);
          a = fmaf(q1.x, kf[4], a); a = fmaf(q1.y, kf[5], a);
          a = fmaf(q1.z, kf[6], a); a = fmaf(q1.w, kf[7], a);
          acc[u] = a;
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kMaxGroup / 2; ++u) {
      const int h = (tid >> 6) + 2 * u;
      if (h < G) S.p[h][j] = j < nv ? acc[u] + gv[u] * sv_raw : -INFINITY;
    }
  }
  __syncthreads();

  // ---- per head: chunk max and weights; warp h writes the head's m and l ----
  for (int h = warp; h < G; h += kThreads / 32) {
    const float z0 = S.p[h][lane], z1 = S.p[h][lane + 32];
    float mc = fmaxf(z0, z1);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mc = fmaxf(mc, __shfl_xor_sync(0xFFFFFFFFu, mc, off));
    // mc is finite: row 0 of every chunk is valid
    const float p0 = tg::exp2_approx(z0 - mc), p1 = tg::exp2_approx(z1 - mc);
    S.p[h][lane] = p0;
    S.p[h][lane + 32] = p1;
    float lc = p0 + p1;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) lc += __shfl_xor_sync(0xFFFFFFFFu, lc, off);
    if (lane == 0) {
      float* pr = partial + ((static_cast<int64_t>(b) * n_hq + kvh * G + h) * n_split + split) * kPartial;
      pr[kDh] = mc;
      pr[kDh + 1] = lc;
    }
  }
  __syncthreads();

  // ---- o = sum_j p_j v_j ----
#pragma unroll 4
  for (int jj = 0; jj < nv; ++jj) {
    const uint32_t vv = *reinterpret_cast<const uint32_t*>(vt + sw_off(jj, e));
    const float v0 = bf16_lo(vv), v1 = bf16_hi(vv);
#pragma unroll
    for (int u = 0; u < kMaxGroup / 2; ++u) {
      const int h = (tid >> 6) + 2 * u;
      if (h < G) {
        const float pj = S.p[h][jj];
        o0[u] = fmaf(pj, v0, o0[u]);
        o1[u] = fmaf(pj, v1, o1[u]);
      }
    }
  }
#pragma unroll
  for (int u = 0; u < kMaxGroup / 2; ++u) {
    const int h = (tid >> 6) + 2 * u;
    if (h < G) {
      float* pr = partial + ((static_cast<int64_t>(b) * n_hq + kvh * G + h) * n_split + split) * kPartial;
      *reinterpret_cast<float2*>(pr + e) = make_float2(o0[u], o1[u]);
    }
  }
}

// Merge one row's chunk partials. Chunks come in blocks of 128: thread d of group 0
// loads chunk d's max and sum into shared memory, every thread takes the block's
// max, and group g (threads 128g .. 128g + 127, thread d of it owning output
// dimension d) folds the block's chunks 32g .. 32g + 31 with all 32 loads in
// flight. Every group scales by the same running max, so the groups' sums add at
// the end.
constexpr int kCombineBlock = 32;
constexpr int kCombineGroups = 4;
constexpr int kCombineThreads = kCombineGroups * kDh;

__global__ void __launch_bounds__(kCombineThreads)
    decode_combine_kernel(const float* __restrict__ partial, const int32_t* __restrict__ cache_len,
                          int cap, int max_len, int n_hq, int n_split,
                          __nv_bfloat16* __restrict__ out, int* status) {
  __shared__ float sm[kDh], sl[kDh];
  __shared__ float racc[kCombineGroups - 1][kDh], rl[kCombineGroups - 1][kDh];
  tg::pdl_launch_dependents();
  tg::pdl_wait();
  const int hq = blockIdx.x, b = blockIdx.y;
  const int grp = threadIdx.x / kDh, d = threadIdx.x % kDh;
  const int len = cache_len[b];
  __nv_bfloat16* o = out + (static_cast<int64_t>(b) * n_hq + hq) * kDh;
  if (len < 0 || len > cap || len > max_len) {
    if (threadIdx.x == 0 && hq == 0) tg::set_status(status, TG_ERR_DEVICE_CHECK);
    return;
  }
  if (len == 0) {   // an empty cache attends to nothing
    if (grp == 0) o[d] = __float2bfloat16_rn(0.f);
    return;
  }
  const int nsp = (len + kChunk - 1) / kChunk;   // chunks holding a partial
  const float* pr = partial + (static_cast<int64_t>(b) * n_hq + hq) * n_split * kPartial;
  float acc = 0.f, L = 0.f, M = -INFINITY;
  for (int s0 = 0; s0 < nsp; s0 += kDh) {   // blocks of up to 128 chunks (one block below 8k keys)
    const int ns = min(kDh, nsp - s0);
    const int u0 = grp * kCombineBlock;   // this group's 32 chunks of the block
    float v[kCombineBlock];
#pragma unroll
    for (int u = 0; u < kCombineBlock; ++u)
      v[u] = u0 + u < ns ? pr[(s0 + u0 + u) * kPartial + d] : 0.f;
    if (grp == 0 && d < ns) {
      sm[d] = pr[(s0 + d) * kPartial + kDh];
      sl[d] = pr[(s0 + d) * kPartial + kDh + 1];
    }
    __syncthreads();
    float mb = M;
    for (int u = 0; u < ns; ++u) mb = fmaxf(mb, sm[u]);
    const float scale = tg::exp2_approx(M - mb);   // the earlier blocks, onto the new max
    acc *= scale;
    L *= scale;
    M = mb;
#pragma unroll
    for (int u = 0; u < kCombineBlock; ++u) {
      if (u0 + u < ns) {
        const float w = tg::exp2_approx(sm[u0 + u] - M);
        L = fmaf(w, sl[u0 + u], L);
        acc = fmaf(w, v[u], acc);
      }
    }
    __syncthreads();   // sm, sl are rewritten by the next block
  }
  if (grp > 0) {
    racc[grp - 1][d] = acc;
    rl[grp - 1][d] = L;
  }
  __syncthreads();
  if (grp == 0) {
#pragma unroll
    for (int g = 0; g < kCombineGroups - 1; ++g) {
      acc += racc[g][d];
      L += rl[g][d];
    }
    o[d] = __float2bfloat16_rn(acc / L);
  }
}

__global__ void __launch_bounds__(kThreads)
    cache_append_kernel(const uint4* __restrict__ k_new, const uint4* __restrict__ v_new,
                        const float* __restrict__ s_new, int cap, int row_vecs,
                        uint4* __restrict__ k_cache, uint4* __restrict__ v_cache,
                        float* __restrict__ s_cache, int32_t* __restrict__ cache_len, int* status) {
  tg::pdl_launch_dependents();
  tg::pdl_wait();
  const int b = blockIdx.x;
  const int len = cache_len[b];
  if (len < 0 || len >= cap) {   // full (or corrupt) cache: nothing is written
    if (threadIdx.x == 0) tg::set_status(status, TG_ERR_DEVICE_CHECK);
    return;
  }
  const int64_t dst = (static_cast<int64_t>(b) * cap + len) * row_vecs;
  const int64_t cache_vecs = static_cast<int64_t>(gridDim.x) * cap * row_vecs;
  for (int i = threadIdx.x; i < row_vecs; i += kThreads) {
    if (!tg::in_bounds(dst + i, cache_vecs, status)) break;
    k_cache[dst + i] = k_new[static_cast<int64_t>(b) * row_vecs + i];
    v_cache[dst + i] = v_new[static_cast<int64_t>(b) * row_vecs + i];
  }
  __syncthreads();   // every thread has read cache_len[b] before it moves
  if (threadIdx.x == 0 &&
      tg::in_bounds(static_cast<int64_t>(b) * cap + len, static_cast<int64_t>(gridDim.x) * cap, status)) {
    s_cache[static_cast<int64_t>(b) * cap + len] = s_new[b];
    cache_len[b] = len + 1;
  }
}

inline int n_splits(int max_len) { return (max_len + kChunk - 1) / kChunk; }

}  // namespace

extern "C" size_t tg_gated_decode_workspace_size(int batch, int n_hq, int head_dim, int max_len) {
  if (batch <= 0 || n_hq <= 0 || head_dim != kDh || max_len <= 0) return 0;
  return static_cast<size_t>(batch) * n_hq * n_splits(max_len) * kPartial * sizeof(float);
}

extern "C" tg_status tg_cache_append(const void* k_new, const void* v_new, const float* s_new,
                                     int batch, int cap, int n_hkv, int head_dim, void* k_cache,
                                     void* v_cache, float* s_cache, int32_t* cache_len,
                                     tg_stream_t stream) {
  tg::NvtxRange nvtx_range("tg_cache_append");
  if (batch < 0 || cap <= 0 || n_hkv <= 0 || head_dim <= 0) return TG_ERR_INVALID_ARG;
  if (batch == 0) return TG_OK;
  if (!k_new || !v_new || !s_new || !k_cache || !v_cache || !s_cache || !cache_len)
    return TG_ERR_INVALID_ARG;
  if (head_dim != kDh || batch > 65535) return TG_ERR_UNSUPPORTED;
  if (!tg::aligned16(k_new) || !tg::aligned16(v_new) || !tg::aligned16(k_cache) ||
      !tg::aligned16(v_cache))
    return TG_ERR_MISALIGNED;
  int* st = tg::status_word();
  if (!st) return TG_ERR_CUDA;
  const int row_vecs = n_hkv * kDh * 2 / 16;
  return tg::launch(cache_append_kernel, dim3(batch), dim3(kThreads), 0, stream, 0,
                    static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new), s_new, cap,
                    row_vecs, static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), s_cache,
                    cache_len, st);
}

extern "C" tg_status tg_gated_decode(const void* q, const void* k_cache, const void* v_cache,
                                     const float* s_cache, const int32_t* cache_len, int batch,
                                     int cap, int max_len, int n_hq, int n_hkv, int head_dim,
                                     const float* gain, const float* tau, void* out,
                                     void* workspace, size_t workspace_bytes,
                                     tg_stream_t stream) {
  tg::NvtxRange nvtx_range("tg_gated_decode");
  if (batch < 0 || cap <= 0 || max_len < 0 || n_hq <= 0 || n_hkv <= 0 || head_dim <= 0)
    return TG_ERR_INVALID_ARG;
  if (batch == 0) return TG_OK;
  if (!q || !k_cache || !v_cache || !s_cache || !cache_len || !gain || !tau || !out)
    return TG_ERR_INVALID_ARG;
  if (n_hq % n_hkv != 0) return TG_ERR_INVALID_ARG;
  if (max_len > cap) return TG_ERR_INVALID_ARG;
  if (head_dim != kDh || n_hq / n_hkv > kMaxGroup) return TG_ERR_UNSUPPORTED;
  if (n_hq > 65535 || n_hkv > 65535 || batch > 65535) return TG_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(batch) * cap > INT32_MAX - kChunk) return TG_ERR_UNSUPPORTED;
  if (!tg::aligned16(q) || !tg::aligned16(k_cache) || !tg::aligned16(v_cache) ||
      !tg::aligned16(out))
    return TG_ERR_MISALIGNED;
  const int ns = n_splits(max_len > 0 ? max_len : 1);
  const size_t need = tg_gated_decode_workspace_size(batch, n_hq, head_dim, max_len > 0 ? max_len : 1);
  if (!workspace || workspace_bytes < need) return TG_ERR_WORKSPACE;
  if (!tg::aligned16(workspace)) return TG_ERR_MISALIGNED;
  int* st = tg::status_word();
  if (!st) return TG_ERR_CUDA;
  CUtensorMap tk, tv;
  const uint64_t dims[3] = {kDh, static_cast<uint64_t>(n_hkv), static_cast<uint64_t>(batch) * cap};
  const uint64_t strides[2] = {kDh * 2, static_cast<uint64_t>(n_hkv) * kDh * 2};
  const uint32_t box[3] = {64, 1, kChunk};
  if (!tg::encode_tmap(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, k_cache, dims, strides, box,
                       CU_TENSOR_MAP_SWIZZLE_128B) ||
      !tg::encode_tmap(&tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, v_cache, dims, strides, box,
                       CU_TENSOR_MAP_SWIZZLE_128B))
    return TG_ERR_CUDA;
  if (!tg::ensure_smem(reinterpret_cast<const void*>(decode_split_kernel), static_cast<int>(kDecodeSmem)))
    return TG_ERR_CUDA;
  float* part = static_cast<float*>(workspace);
  tg_status r = TG_OK;
  if (max_len > 0) {
    r = tg::launch(decode_split_kernel, dim3(ns, n_hkv, batch), dim3(kThreads), kDecodeSmem, stream, 0,
                   tk, tv, static_cast<const __nv_bfloat16*>(q), s_cache, cache_len, cap, max_len,
                   n_hq, n_hkv, gain, tau, part, ns, st);
    if (r != TG_OK) return r;
  }
  return tg::launch(decode_combine_kernel, dim3(n_hq, batch), dim3(kCombineThreads), 0, stream, 0,
                    static_cast<const float*>(part), cache_len, cap, max_len, n_hq, ns,
                    static_cast<__nv_bfloat16*>(out), st);
}

// ---- decode with library-owned scratch, for callers that cannot allocate ----
//
// tg_gated_decode needs a caller-provided workspace for its per-chunk partial
// results. Some callers cannot allocate one where they call decode: a host
// program whose device memory all belongs to another runtime's pool (so a
// library may not, or cannot, call cudaMalloc behind it), or a token-by-token
// generation loop that must not allocate at all because cudaMalloc and cudaFree
// can synchronise the whole device. tg_gated_decode_noalloc serves them from a
// fixed array in the library's own device memory instead. Every device that
// loads the library holds that array (TG_DECODE_NOALLOC_SCRATCH_BYTES) until the
// process exits, whether or not this entry point is ever called.
static __device__ __align__(256) float g_decode_scratch[TG_DECODE_NOALLOC_SCRATCH_BYTES / sizeof(float)];

namespace {

constexpr int kMaxScratchDevices = 64;
float* g_scratch_addr[kMaxScratchDevices];   // device address of the array, per device
std::mutex g_scratch_mu;

// In host code g_decode_scratch names a host-side stand-in, not device memory: the
// array's address on the current device comes from the runtime, looked up once
// per device (with that device current) and kept.
float* decode_scratch_on_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxScratchDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) return nullptr;
    g_scratch_addr[dev] = static_cast<float*>(p);
  }
  return g_scratch_addr[dev];
}

}  // namespace

extern "C" tg_status tg_gated_decode_noalloc(const void* q, const void* k_cache,
                                             const void* v_cache, const float* s_cache,
                                             const int32_t* cache_len, int batch, int cap,
                                             int max_len, int n_hq, int n_hkv, int head_dim,
                                             const float* gain, const float* tau, void* out,
                                             tg_stream_t stream) {
  tg::NvtxRange nvtx_range("tg_gated_decode_noalloc");
  if (batch > 0 && n_hq > 0 && head_dim > 0) {
    const size_t need = tg_gated_decode_workspace_size(batch, n_hq, head_dim, max_len > 0 ? max_len : 1);
    if (need > TG_DECODE_NOALLOC_SCRATCH_BYTES) return TG_ERR_WORKSPACE;   // beyond the fixed array
  }
  float* scratch = nullptr;
  if (batch > 0) {
    scratch = decode_scratch_on_current_device();
    if (!scratch) return TG_ERR_CUDA;
  }
  return tg_gated_decode(q, k_cache, v_cache, s_cache, cache_len, batch, cap, max_len, n_hq, n_hkv,
                         head_dim, gain, tau, out, scratch, TG_DECODE_NOALLOC_SCRATCH_BYTES, stream);
}

// tg_gate_score: the gate MLP scorer (MarkTechPost page on TokenGate, section
// "Comment TokenGate a-t-il appris le fonctionnement de la réduction des tokens
// ?": a small MLP scores each token from its post-attention residual at layer L).
//     s_i = b2 + sum_k w2[k] * GELU(b1[k] + x_i . w1[k,:])
//
// bf16 path: one CTA per 128-token tile computes the whole hidden layer
// (M=128 tokens x N=h units x K=d) with tcgen05.mma (kind::f16, f32 accumulate)
// into two 128 x h fp32 accumulators in tensor memory, one per half of the
// reduction (d/2 columns each, accumulated in a fixed order). Even CTAs run the
// first half first, odd CTAs the second, so at any moment only half of the CTAs
// read the same w1 tile (every CTA reads all of w1, from L2); the epilogue adds
// the two accumulators in a fixed order, so a token's score does not depend on
// which CTA computed it. A TMA producer thread streams
// 128x64 tiles of x and hx64 tiles of w1 (128-byte swizzle) through a 4-stage
// mbarrier ring; one MMA thread issues 4 K=16 MMAs per stage and frees the stage
// with tcgen05.commit. The epilogue never leaves fp32: 16 warps read the
// accumulator (warp w: lanes 32*(w%4).., a quarter of the columns), add b1, apply
// erf-GELU and dot with w2; the four column partials are summed in a fixed
// order, so a token's score depends only on its own row. The GELU's erf is the
// Abramowitz-Stegun 7.1.26 form (|error| <= 1.5e-7), branch-free.
//
// When there are more 128-token tiles than SMs, a 256-token variant runs instead:
// two row tiles per CTA share every w1 stage (two MMAs per K step into two
// accumulators), which halves the w1 bytes each token costs.
//
// f32 path: an exact fp32 SIMT kernel (one CTA per token) for small checks.
#include "common.cuh"

namespace {

constexpr int kBM = 128;      // tokens per tile
constexpr int kBK = 64;       // reduction columns per stage (128 bytes of bf16)
constexpr int kStages = 4;
constexpr int kThreads = 512;

template <int H>
struct GateSmem {
  uint8_t a[kStages][kBM * kBK * 2];   // x tiles, 16 KB each
  uint8_t b[kStages][H * kBK * 2];     // w1 tiles
  float b1[H];
  float w2[H];
  float part[4][kBM];
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t acc_full;
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ float gelu_erf(float u) {
  return 0.5f * u * (1.0f + erff(u * 0.70710678118654752f));
}

// erf by Abramowitz & Stegun, Handbook of Mathematical Functions, eq. 7.1.26
// (Hastings' rational form): for x >= 0,
//     erf(x) = 1 - (a1 t + a2 t^2 + a3 t^3 + a4 t^4 + a5 t^5) exp(-x^2),  t = 1/(1 + p x),
// with |error| <= 1.5e-7; erf is odd. Branch-free, one MUFU reciprocal and one MUFU
// exp2 per call, which is what lets 128 x h GELUs per tile fit in the epilogue.
constexpr float kAsP = 0.3275911f;
constexpr float kAsA1 = 0.254829592f;
constexpr float kAsA2 = -0.284496736f;
constexpr float kAsA3 = 1.421413741f;
constexpr float kAsA4 = -1.453152027f;
constexpr float kAsA5 = 1.061405429f;

__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

__device__ __forceinline__ float erf_as(float x) {
  const float ax = fabsf(x);
  const float t = rcp_approx(fmaf(kAsP, ax, 1.0f));
  const float poly = t * fmaf(fmaf(fmaf(fmaf(kAsA5, t, kAsA4), t, kAsA3), t, kAsA2), t, kAsA1);
  const float e = tg::exp2_approx(-(ax * ax) * 1.4426950408889634f);
  return copysignf(fmaf(-poly, e, 1.0f), x);
}

// GELU(u) = u Phi(u) = u (1 + erf(u / sqrt 2)) / 2 with the erf above (bf16 path)
__device__ __forceinline__ float gelu_as(float u) {
  return 0.5f * u * (1.0f + erf_as(u * 0.70710678118654752f));
}

template <int H>
__global__ void __launch_bounds__(kThreads, 1)
    gate_bf16_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                     const float* __restrict__ b1, const float* __restrict__ w2, float b2,
                     int64_t n_tokens, int d, float* __restrict__ scores, int* status) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (tg::smem_u32(smem_raw) & 1023u)) & 1023u;
  GateSmem<H>& S = *reinterpret_cast<GateSmem<H>*>(smem_raw + pad);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t m0 = static_cast<int64_t>(blockIdx.x) * kBM;
  const int nk = d / kBK;
  const int half = nk / 2;                               // k-blocks [0, half) -> accumulator 0
  const int kstart = (blockIdx.x & 1) ? half : 0;       // odd CTAs start with the second half
  auto kblock = [&](int i) { const int k = i + kstart; return k < nk ? k : k - nk; };

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
    tg::tmem_alloc(&S.tmem_base, 2 * H);
    tg::tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tg::tma_prefetch_desc(&tm_x);
    tg::tma_prefetch_desc(&tm_w);
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
      tg::mbar_arrive_expect_tx(&S.full[s], (kBM + H) * kBK * 2);
      tg::tma_load_2d(S.a[s], &tm_x, &S.full[s], kblock(kb) * kBK, static_cast<int>(m0));
      tg::tma_load_2d(S.b[s], &tm_w, &S.full[s], kblock(kb) * kBK, 0);
      ++issued;
    }
    if (S.abort_flag) {   // let copies already in flight land before the CTA can exit
      for (int kb = issued > kStages ? issued - kStages : 0; kb < issued; ++kb)
        tg::mbar_wait(&S.full[kb % kStages], (kb / kStages) & 1, status, nullptr);
    }
  } else if (warp == 1 && lane == 0) {
    // ---- MMA issuer ----
    constexpr uint32_t idesc = tg::idesc_bf16_f32(kBM, H, false, false);
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % kStages;
      if (!tg::mbar_wait(&S.full[s], (kb / kStages) & 1, status, &S.abort_flag)) break;
      tg::tc_fence_after();
      const uint32_t a0 = tg::smem_u32(S.a[s]), b0 = tg::smem_u32(S.b[s]);
      const int kg = kblock(kb);
      const uint32_t acc = kg < half ? tmem : tmem + H;     // accumulator of this k-block
      const bool first = (kg == 0) || (kg == half);         // first k-block of its half
#pragma unroll
      for (int k = 0; k < kBK / 16; ++k) {
        tg::mma_bf16_ss(acc, tg::smem_desc_sw128(a0 + 32 * k, 16, 1024),
                        tg::smem_desc_sw128(b0 + 32 * k, 16, 1024), idesc, !first || k != 0);
      }
      tg::mma_commit(&S.empty[s]);
    }
    tg::mma_commit(&S.acc_full);
  } else if (warp >= 2) {
    // stage the epilogue's constants while the mainloop runs
    for (int i = tid - 64; i < H; i += kThreads - 64) {
      S.b1[i] = b1[i];
      S.w2[i] = w2[i];
    }
  }
  __syncwarp();
  tg::named_barrier(1, kThreads);   // b1/w2 staged; producer and MMA loops issued

  // ---- epilogue: all 16 warps ----
  constexpr int kCols = H / 4;               // accumulator columns per warp
  const int lg = warp & 3, cgp = warp >> 2;
  const int row = lg * 32 + lane;
  float acc = 0.f;
  const bool ok = tg::mbar_wait(&S.acc_full, 0, status, &S.abort_flag);
  if (ok) {
    tg::tc_fence_after();
    uint32_t r[kCols], r2[kCols];
    const uint32_t lrow = static_cast<uint32_t>(lg * 32) << 16;
#pragma unroll
    for (int c = 0; c < kCols; c += 16) {
      tg::tmem_ld16(tmem + lrow + cgp * kCols + c, r + c);
      tg::tmem_ld16(tmem + H + lrow + cgp * kCols + c, r2 + c);
    }
    tg::tmem_ld_wait();
    float a2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < kCols; ++j) {
      const int col = cgp * kCols + j;
      // accumulator 0 is empty when there is a single k-block (half == 0)
      const float u = (half > 0 ? __uint_as_float(r[j]) : 0.f) + __uint_as_float(r2[j]);
      a2[j & 3] = fmaf(S.w2[col], gelu_as(u + S.b1[col]), a2[j & 3]);
    }
    acc = (a2[0] + a2[1]) + (a2[2] + a2[3]);
  }
  S.part[cgp][row] = acc;
  tg::tc_fence_before();
  __syncthreads();
  if (tid < kBM) {
    const float s = b2 + ((S.part[0][tid] + S.part[1][tid]) + (S.part[2][tid] + S.part[3][tid]));
    if (m0 + tid < n_tokens) scores[m0 + tid] = s;
  }
  if (warp == 2) {
    tg::tc_fence_after();
    tg::tmem_dealloc(tmem, 2 * H);
  }
}

// 256-token variant, used when there are more 128-token tiles than SMs: every
// CTA streams all of w1, so a CTA that owns two row tiles halves the w1 bytes per
// token. Each stage holds two 128x64 x tiles and one hx64 w1 tile; per K=16 step
// the MMA thread issues one MMA per row tile into its own 128 x h accumulator (2h
// TMEM columns in all), both with the same w1 operand. Every accumulator is
// summed over d in one fixed order, so a token's score depends only on its row.
constexpr int kPairSmemBudget = 196608;   // bytes of x + w1 stages

template <int H>
struct GatePair {
  static constexpr int kStageBytes = 2 * kBM * kBK * 2 + H * kBK * 2;
  static constexpr int kStages = kPairSmemBudget / kStageBytes > 6 ? 6 : kPairSmemBudget / kStageBytes;
};

template <int H>
struct GatePairSmem {
  uint8_t a[GatePair<H>::kStages][2][kBM * kBK * 2];   // two x tiles, 16 KB each
  uint8_t b[GatePair<H>::kStages][H * kBK * 2];        // w1 tile
  float b1[H];
  float w2[H];
  float part[2][4][kBM];
  uint64_t full[GatePair<H>::kStages];
  uint64_t empty[GatePair<H>::kStages];
  uint64_t acc_full;
  uint32_t tmem_base;
  int abort_flag;
};

template <int H>
__global__ void __launch_bounds__(kThreads, 1)
    gate_bf16_pair_kernel(const __grid_constant__ CUtensorMap tm_x,
                          const __grid_constant__ CUtensorMap tm_w, const float* __restrict__ b1,
                          const float* __restrict__ w2, float b2, int64_t n_tokens, int d,
                          float* __restrict__ scores, int* status) {
  constexpr int kS = GatePair<H>::kStages;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (tg::smem_u32(smem_raw) & 1023u)) & 1023u;
  GatePairSmem<H>& S = *reinterpret_cast<GatePairSmem<H>*>(smem_raw + pad);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t m0 = static_cast<int64_t>(blockIdx.x) * (2 * kBM);
  const int nk = d / kBK;

  if (tid == 0) {
    for (int s = 0; s < kS; ++s) {
      tg::mbar_init(&S.full[s], 1);
      tg::mbar_init(&S.empty[s], 1);
    }
    tg::mbar_init(&S.acc_full, 1);
    S.abort_flag = 0;
    tg::fence_barrier_init();
  }
  if (warp == 2) {
    tg::tmem_alloc(&S.tmem_base, 2 * H);
    tg::tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tg::tma_prefetch_desc(&tm_x);
    tg::tma_prefetch_desc(&tm_w);
  }
  tg::tc_fence_before();
  __syncthreads();
  tg::tc_fence_after();
  const uint32_t tmem = S.tmem_base;
  tg::pdl_launch_dependents();
  tg::pdl_wait();   // global memory only from here on

  if (warp == 0 && lane == 0) {
    // ---- TMA producer: two x tiles and the shared w1 tile per stage ----
    int issued = 0;
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % kS;
      if (kb >= kS && !tg::mbar_wait(&S.empty[s], ((kb / kS) - 1) & 1, status, &S.abort_flag))
        break;
      tg::mbar_arrive_expect_tx(&S.full[s], GatePair<H>::kStageBytes);
      tg::tma_load_2d(S.a[s][0], &tm_x, &S.full[s], kb * kBK, static_cast<int>(m0));
      tg::tma_load_2d(S.a[s][1], &tm_x, &S.full[s], kb * kBK, static_cast<int>(m0 + kBM));
      tg::tma_load_2d(S.b[s], &tm_w, &S.full[s], kb * kBK, 0);
      ++issued;
    }
    if (S.abort_flag) {   // let copies already in flight land before the CTA can exit
      for (int kb = issued > kS ? issued - kS : 0; kb < issued; ++kb)
        tg::mbar_wait(&S.full[kb % kS], (kb / kS) & 1, status, nullptr);
    }
  } else if (warp == 1 && lane == 0) {
    // ---- MMA issuer: per K=16 step one MMA per row tile, same w1 operand ----
    constexpr uint32_t idesc = tg::idesc_bf16_f32(kBM, H, false, false);
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % kS;
      if (!tg::mbar_wait(&S.full[s], (kb / kS) & 1, status, &S.abort_flag)) break;
      tg::tc_fence_after();
      const uint32_t a0 = tg::smem_u32(S.a[s][0]), a1 = tg::smem_u32(S.a[s][1]);
      const uint32_t b0 = tg::smem_u32(S.b[s]);
#pragma unroll
      for (int k = 0; k < kBK / 16; ++k) {
        const uint64_t bdesc = tg::smem_desc_sw128(b0 + 32 * k, 16, 1024);
        const uint32_t acc = (kb > 0 || k > 0) ? 1u : 0u;
        tg::mma_bf16_ss(tmem, tg::smem_desc_sw128(a0 + 32 * k, 16, 1024), bdesc, idesc, acc);
        tg::mma_bf16_ss(tmem + H, tg::smem_desc_sw128(a1 + 32 * k, 16, 1024), bdesc, idesc, acc);
      }
      tg::mma_commit(&S.empty[s]);
    }
    tg::mma_commit(&S.acc_full);
  } else if (warp >= 2) {
    for (int i = tid - 64; i < H; i += kThreads - 64) {
      S.b1[i] = b1[i];
      S.w2[i] = w2[i];
    }
  }
  __syncwarp();
  tg::named_barrier(1, kThreads);   // b1/w2 staged; producer and MMA loops issued

  // ---- epilogue: all 16 warps, the two row tiles one after the other ----
  constexpr int kCols = H / 4;
  const int lg = warp & 3, cgp = warp >> 2;
  const int row = lg * 32 + lane;
  const bool ok = tg::mbar_wait(&S.acc_full, 0, status, &S.abort_flag);
  if (ok) tg::tc_fence_after();
  const uint32_t lrow = static_cast<uint32_t>(lg * 32) << 16;
#pragma unroll 1
  for (int rt = 0; rt < 2; ++rt) {
    float acc = 0.f;
    if (ok) {
      uint32_t r[kCols];
#pragma unroll
      for (int c = 0; c < kCols; c += 16) tg::tmem_ld16(tmem + rt * H + lrow + cgp * kCols + c, r + c);
      tg::tmem_ld_wait();
      float a2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int j = 0; j < kCols; ++j) {
        const int col = cgp * kCols + j;
        a2[j & 3] = fmaf(S.w2[col], gelu_as(__uint_as_float(r[j]) + S.b1[col]), a2[j & 3]);
      }
      acc = (a2[0] + a2[1]) + (a2[2] + a2[3]);
    }
    S.part[rt][cgp][row] = acc;
  }
  tg::tc_fence_before();
  __syncthreads();
  if (tid < 2 * kBM) {
    const int rt = tid / kBM, rr = tid % kBM;
    const float s = b2 + ((S.part[rt][0][rr] + S.part[rt][1][rr]) + (S.part[rt][2][rr] + S.part[rt][3][rr]));
    if (m0 + tid < n_tokens) scores[m0 + tid] = s;
  }
  if (warp == 2) {
    tg::tc_fence_after();
    tg::tmem_dealloc(tmem, 2 * H);
  }
}

// Exact fp32 path: one CTA per token, hidden units strided over the threads,
// fixed-order block reduction.
constexpr int kF32Threads = 128;

__global__ void __launch_bounds__(kF32Threads)
    gate_f32_kernel(const float* __restrict__ x, const float* __restrict__ w1,
                    const float* __restrict__ b1, const float* __restrict__ w2, float b2, int d,
                    int h, float* __restrict__ scores) {
  extern __shared__ float xrow[];
  __shared__ float red[kF32Threads];
  tg::pdl_launch_dependents();
  tg::pdl_wait();
  const int64_t i = blockIdx.x;
  for (int c = threadIdx.x; c < d; c += kF32Threads) xrow[c] = x[i * d + c];
  __syncthreads();
  float part = 0.f;
  for (int k = threadIdx.x; k < h; k += kF32Threads) {
    const float* w = w1 + static_cast<int64_t>(k) * d;
    float u = 0.f;
    for (int c = 0; c < d; ++c) u = fmaf(xrow[c], w[c], u);
    part += w2[k] * gelu_erf(u + b1[k]);
  }
  red[threadIdx.x] = part;
  __syncthreads();
  for (int o = kF32Threads / 2; o > 0; o >>= 1) {
    if (threadIdx.x < o) red[threadIdx.x] += red[threadIdx.x + o];
    __syncthreads();
  }
  if (threadIdx.x == 0) scores[i] = b2 + red[0];
}

template <int H>
tg_status launch_gate_bf16(const void* x, int64_t n, int d, const void* w1, const float* b1,
                           const float* w2, float b2, float* scores, cudaStream_t st) {
  int* status = tg::status_word();
  if (!status) return TG_ERR_CUDA;
  CUtensorMap tx, tw;
  const uint64_t dx[2] = {static_cast<uint64_t>(d), static_cast<uint64_t>(n)};
  const uint64_t sx[1] = {static_cast<uint64_t>(d) * 2};
  const uint32_t bx[2] = {kBK, kBM};
  const uint64_t dw[2] = {static_cast<uint64_t>(d), static_cast<uint64_t>(H)};
  const uint32_t bw[2] = {kBK, H};
  if (!tg::encode_tmap(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, x, dx, sx, bx,
                       CU_TENSOR_MAP_SWIZZLE_128B) ||
      !tg::encode_tmap(&tw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, w1, dw, sx, bw,
                       CU_TENSOR_MAP_SWIZZLE_128B))
    return TG_ERR_CUDA;
  const int64_t tiles = (n + kBM - 1) / kBM;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return TG_ERR_CUDA;
  if (tiles > sms) {   // more tiles than SMs: two row tiles per CTA, w1 streamed once for both
    const size_t smem = sizeof(GatePairSmem<H>) + 1024;
    if (!tg::ensure_smem(reinterpret_cast<const void*>(gate_bf16_pair_kernel<H>),
                         static_cast<int>(smem)))
      return TG_ERR_CUDA;
    return tg::launch(gate_bf16_pair_kernel<H>, dim3(static_cast<unsigned>((tiles + 1) / 2)),
                      dim3(kThreads), smem, st, 0, tx, tw, b1, w2, b2, n, d, scores, status);
  }
  const size_t smem = sizeof(GateSmem<H>) + 1024;
  if (!tg::ensure_smem(reinterpret_cast<const void*>(gate_bf16_kernel<H>), static_cast<int>(smem)))
    return TG_ERR_CUDA;
  return tg::launch(gate_bf16_kernel<H>, dim3(static_cast<unsigned>(tiles)), dim3(kThreads), smem, st,
                    0, tx, tw, b1, w2, b2, n, d, scores, status);
}

}  // namespace

extern "C" tg_status tg_gate_score(const void* x, tg_dtype dtype, int64_t n_tokens, int d,
                                   const void* w1, const float* b1, const float* w2, float b2,
                                   int h, float* scores, tg_stream_t stream) {
  tg::NvtxRange nvtx_range("tg_gate_score");
  if (n_tokens < 0 || d <= 0 || h <= 0) return TG_ERR_INVALID_ARG;
  if (n_tokens == 0) return TG_OK;
  if (!x || !w1 || !b1 || !w2 || !scores) return TG_ERR_INVALID_ARG;
  if (dtype == TG_BF16) {
    if (d % kBK != 0 || (h != 64 && h != 128 && h != 256)) return TG_ERR_UNSUPPORTED;
    if (n_tokens > INT32_MAX - kBM) return TG_ERR_UNSUPPORTED;
    if (!tg::aligned16(x) || !tg::aligned16(w1)) return TG_ERR_MISALIGNED;
    switch (h) {
      case 64: return launch_gate_bf16<64>(x, n_tokens, d, w1, b1, w2, b2, scores, stream);
      case 128: return launch_gate_bf16<128>(x, n_tokens, d, w1, b1, w2, b2, scores, stream);
      default: return launch_gate_bf16<256>(x, n_tokens, d, w1, b1, w2, b2, scores, stream);
    }
  }
  if (dtype == TG_F32) {
    if (h > 1024 || d > 12288) return TG_ERR_UNSUPPORTED;
    if (n_tokens > INT32_MAX) return TG_ERR_UNSUPPORTED;
    return tg::launch(gate_f32_kernel, dim3(static_cast<unsigned>(n_tokens)), dim3(kF32Threads),
                      static_cast<size_t>(d) * 4, stream, 0, static_cast<const float*>(x),
                      static_cast<const float*>(w1), b1, w2, b2, d, h, scores);
  }
  return TG_ERR_UNSUPPORTED;
}

// tg_select_topk: top-K of the droppable document span with the question always
// kept (MarkTechPost page on TokenGate, section "Comment TokenGate a-t-il appris
// le fonctionnement de la réduction des tokens ?": a top-K selector keeps the
// best-scoring tokens; only the document part may be dropped; section "Comment
// déployer TokenGate ?": {state} marks the document, max_kept_prefill_tokens the
// budget).
//
// One thread-block cluster per sequence, one launch for the whole batch. The
// cluster has enough CTAs (1..16, where the device runs 16-CTA clusters, else
// 1..8) for about 2048 keys each (at most 24576), so the passes below stay short.
// Each CTA holds a contiguous slice of the sequence in shared memory twice: the raw fp32 scores (for the kept-score output) and
// order-preserving 32-bit keys (NaN lowest, -0 == +0). Tokens outside the
// document (and padding) get key 0; their count is subtracted from bin 0 so the
// histograms see document tokens only.
//
// A 4-pass MSB-first radix select (8-bit digits) finds the exact K-th largest
// document key T: per-warp histograms fed by 128-bit shared loads (4 keys per
// lane), summed per CTA and across the cluster through distributed shared memory,
// and the digit holding the K-th key found with a block suffix scan. Emission
// keeps every token outside the span, every document token with key > T, and the
// `need` lowest-positioned document tokens with key == T (ties to the lower
// position). One counting pass gives each warp's tie count and tie-independent
// kept count; since the ties kept before any point number min(need, ties before
// it), one exchange of those two counts through distributed shared memory fixes
// every CTA's and warp's output offset, and a second pass writes the kept rows
// in order (ranks from warp scans), with their scores and their positions within
// the sequence. No global scratch.
#include <cooperative_groups.h>

#include <mutex>

#include "common.cuh"

namespace cg = cooperative_groups;

namespace {

constexpr int kMaxCluster = 16;     // 16 where the device runs such clusters (else 8)
constexpr int kPortableCluster = 8;
constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kKeysTarget = 2048;                                    // keys per CTA aimed at
constexpr int kMaxKeysPerCta = TG_SELECT_MAX_SEQLEN / kPortableCluster;   // 24576
constexpr int kChunkQuant = kWarps * 128;                            // 128 keys per warp step

struct alignas(16) SelectSmem {
  uint32_t whist[kWarps][256];   // per-warp histograms
  uint32_t hist[2][256];         // this CTA's histogram, by pass parity (read by peers)
  uint32_t scan[8];
  uint32_t warp_tot[kWarps];
  uint32_t warp_base[kWarps];
  uint32_t warp_off[kWarps];
  uint32_t warp_eq_off[kWarps];
  uint32_t cta_eq;               // published to peers
  uint32_t cta_keep;             // published to peers
  uint32_t digit;
  uint32_t remaining;
  uint32_t seq_keep;
  int64_t red[kWarps];
  // followed by: uint32_t keys[chunk]; float raw[chunk];
};

inline int select_cluster(int max_len, int max_cluster) {
  int c = (max_len + kKeysTarget - 1) / kKeysTarget;
  if (c < 1) c = 1;
  if (c > max_cluster) c = max_cluster;
  return c;
}

inline int select_chunk(int max_len, int csize) {
  int c = (max_len + csize - 1) / csize;
  c = (c + kChunkQuant - 1) / kChunkQuant * kChunkQuant;
  return c < kChunkQuant ? kChunkQuant : c;
}

__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7FFFFFFFu) > 0x7F800000u) return 0u;   // NaN ranks lowest
  if (u == 0x80000000u) u = 0u;                     // -0 is +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// kept count of a sequence from the (possibly hostile) device arrays, clamped
__device__ __forceinline__ int64_t seq_kept(const int32_t* cu, const int32_t* db,
                                            const int32_t* de, const int32_t* kd, int b) {
  int64_t len = (int64_t)cu[b + 1] - cu[b];
  if (len < 0) len = 0;
  int64_t s0 = db[b], s1 = de[b];
  if (s0 < 0) s0 = 0;
  if (s1 > len) s1 = len;
  int64_t nd = s1 > s0 ? s1 - s0 : 0;
  int64_t k = kd[b];
  if (k < 0) k = 0;
  if (k > nd) k = nd;
  return len - nd + k;
}

__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, v, o);
    if (lane >= o) v += y;
  }
  return v;
}

__device__ __forceinline__ uint32_t key_at(const uint4& k, int e) {
  return e == 0 ? k.x : e == 1 ? k.y : e == 2 ? k.z : k.w;
}

__global__ void __launch_bounds__(kThreads, 1)
    select_topk_kernel(const float* __restrict__ scores, const int32_t* __restrict__ cu_seqlens,
                       const int32_t* __restrict__ doc_begin, const int32_t* __restrict__ doc_end,
                       const int32_t* __restrict__ k_doc, int batch, int64_t total_tokens,
                       int64_t total_kept, int chunk, int32_t* __restrict__ kept_idx, float* __restrict__ kept_scores,
                       int32_t* __restrict__ kept_pos, int32_t* __restrict__ cu_kept,
                       int* status) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  SelectSmem& S = *reinterpret_cast<SelectSmem*>(smem_raw);
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem_raw + sizeof(SelectSmem));
  float* raw = reinterpret_cast<float*>(keys + chunk);

  tg::pdl_launch_dependents();
  tg::pdl_wait();
  cg::cluster_group cluster = cg::this_cluster();
  const unsigned rank = cluster.block_rank();
  const unsigned csize = cluster.num_blocks();
  const int b = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const unsigned full = 0xFFFFFFFFu;

  // ---- output offset: the earlier sequences' kept counts (clamped the same way
  //      for every sequence, so a rejected sequence still has a defined extent).
  //      Per-warp sums here; the block sum is read after the next block barrier,
  //      so these loads overlap the score loads ----
  {
    int64_t acc = 0;
    for (int p = tid; p < b; p += kThreads) acc += seq_kept(cu_seqlens, doc_begin, doc_end, k_doc, p);
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(full, acc, o);
    if (lane == 0) S.red[warp] = acc;
  }
  auto block_out_base = [&]() {   // valid after a __syncthreads that follows the sums
    int64_t t = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) t += S.red[w];
    return t;
  };

  // Rejected sequence (or an inconsistent total found below): its output rows
  // get row id -1, score 0 and position -1, and cu_kept still advances by the
  // clamped count, clipped to total_kept, so the kernels that read these outputs
  // next see in-range offsets and an index the compaction rejects.
  auto reject = [&](int64_t out_base, int64_t count) {
    const int64_t o0 = out_base < total_kept ? out_base : total_kept;
    const int64_t o1 = out_base + count < total_kept ? out_base + count : total_kept;
    for (int64_t r = o0 + (int64_t)rank * kThreads + tid; r < o1; r += (int64_t)csize * kThreads) {
      if (!tg::in_bounds(r, total_kept, status)) break;
      kept_idx[r] = -1;
      if (kept_scores) kept_scores[r] = 0.f;
      if (kept_pos) kept_pos[r] = -1;
    }
    if (rank == 0 && tid == 0) {
      tg::set_status(status, TG_ERR_DEVICE_CHECK);
      if (b == 0) cu_kept[0] = 0;
      cu_kept[b + 1] = (int32_t)o1;
    }
  };

  // ---- sequence geometry (identical in every CTA of the cluster) ----
  const int64_t base = cu_seqlens[b];
  const int64_t len = (int64_t)cu_seqlens[b + 1] - base;
  const int64_t db = doc_begin[b], de = doc_end[b];
  const bool bad = base < 0 || len < 0 || base + len > total_tokens ||
                   len > (int64_t)chunk * csize || db < 0 || de < db || de > len;
  if (bad) {
    __syncthreads();
    reject(block_out_base(), seq_kept(cu_seqlens, doc_begin, doc_end, k_doc, b));
    return;   // uniform across the cluster: nobody reaches a cluster barrier
  }
  const int64_t nd = de - db;
  int64_t k_eff = k_doc[b];
  if (k_eff < 0) k_eff = 0;
  if (k_eff > nd) k_eff = nd;

  // this CTA's slice [c0, c0 + n_local) and its document part [ld0, ld1) (local)
  const int64_t c0 = (int64_t)rank * chunk;
  const int n_local = (int)(len - c0 < 0 ? 0 : (len - c0 > chunk ? chunk : len - c0));
  auto clampl = [&](int64_t v) { return (int)(v < 0 ? 0 : (v > n_local ? n_local : v)); };
  const int ld0 = clampl(db - c0), ld1 = clampl(de - c0);
  const uint32_t excl_local = (uint32_t)(chunk - (ld1 - ld0));   // keys forced to 0

  // ---- load: raw scores and keys into shared memory; when a radix select is
  //      needed, the first pass's per-warp histograms (digit = key >> 24) are
  //      filled on the way (16 loads in flight per thread) ----
  const bool radix = k_eff > 0 && k_eff < nd;
  {
    uint32_t* wh = S.whist[warp];
#pragma unroll
    for (int i = lane; i < 256; i += 32) wh[i] = 0u;
    __syncwarp();
    for (int i0 = tid; i0 < chunk; i0 += 16 * kThreads) {
      float v[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int i = i0 + u * kThreads;
        v[u] = i < n_local && tg::in_bounds(base + c0 + i, total_tokens, status)
                   ? scores[base + c0 + i]
                   : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int i = i0 + u * kThreads;
        if (i < chunk) {
          const uint32_t key = (i >= ld0 && i < ld1) ? score_key(v[u]) : 0u;
          raw[i] = v[u];
          keys[i] = key;
          if (radix) atomicAdd(&wh[key >> 24], 1u);
        }
      }
    }
  }
  __syncthreads();
  const int64_t out_base = block_out_base();

  const int seg = chunk / kWarps;                 // multiple of 128
  const int seg0 = warp * seg;
  const int nsteps = seg / 128;
  const uint4* k4 = reinterpret_cast<const uint4*>(keys) + seg0 / 4;

  // ---- radix select of the k_eff-th largest document key ----
  uint32_t T, need;
  if (k_eff == 0) {
    T = 0xFFFFFFFFu;   // above every key (the largest key, +inf, is 0xFF800000)
    need = 0;
  } else if (!radix) {
    T = 0u;            // k_eff == nd: everything is kept
    need = (uint32_t)nd;
  } else {
    uint32_t prefix = 0, pmask = 0, remaining = (uint32_t)k_eff;
    for (int pass = 0; pass < 4; ++pass) {
      const int shift = 24 - 8 * pass;
      uint32_t* h = S.hist[pass & 1];
      if (pass > 0) {   // the first pass's histograms were filled by the load
        uint32_t* wh = S.whist[warp];   // zeroed by the previous pass's reduction
        for (int st = 0; st < nsteps; ++st) {
          const uint4 kk = k4[st * 32 + lane];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const uint32_t key = key_at(kk, e);
            if ((key & pmask) == prefix) atomicAdd(&wh[(key >> shift) & 0xFFu], 1u);
          }
        }
        __syncthreads();
      }
      if (tid < 256) {
        uint32_t c = 0;
#pragma unroll 8
        for (int w = 0; w < kWarps; ++w) {
          c += S.whist[w][tid];
          S.whist[w][tid] = 0u;   // ready for the next pass
        }
        if (tid == 0 && prefix == 0) c -= excl_local;   // forced-zero keys are not document keys
        h[tid] = c;
      }
      cluster.sync();   // every CTA's histogram of this pass is complete
      if (tid < 256) {
        // thread t holds digit d = 255 - t; an inclusive prefix over t is the
        // count of matching document keys with digit >= d
        const int d = 255 - tid;
        // every peer's count at once (independent remote loads in flight), then
        // summed in rank order
        uint32_t pc[kMaxCluster];
#pragma unroll
        for (int r = 0; r < kMaxCluster; ++r)
          pc[r] = r < static_cast<int>(csize) ? cluster.map_shared_rank(h, r)[d] : 0u;
        uint32_t cnt = 0;
#pragma unroll
        for (int r = 0; r < kMaxCluster; ++r) cnt += pc[r];
        uint32_t inc = warp_incl_scan(cnt, lane);
        if (lane == 31) S.scan[warp] = inc;
        tg::named_barrier(1, 256);   // warps 0-7 only
        uint32_t woff = 0;
        for (int w = 0; w < warp; ++w) woff += S.scan[w];
        inc += woff;
        const uint32_t exc = inc - cnt;
        if (exc < remaining && remaining <= inc) {
          S.digit = (uint32_t)d;
          S.remaining = remaining - exc;
        }
      }
      __syncthreads();
      prefix |= S.digit << shift;
      pmask |= 0xFFu << shift;
      remaining = S.remaining;
    }
    T = prefix;
    need = remaining;
  }

  // ---- emission, pass 1: per-warp counts of ties (document keys == T) and of
  //      tokens kept regardless of ties (outside the document, or key > T) ----
  {
    uint32_t ceq = 0, cbase = 0;
    for (int st = 0; st < nsteps; ++st) {
      const uint4 kk = k4[st * 32 + lane];
      const int i4 = seg0 + st * 128 + lane * 4;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = i4 + e;
        const bool in_doc = i >= ld0 && i < ld1;
        const uint32_t key = key_at(kk, e);
        ceq += in_doc && key == T;
        cbase += i < n_local && (!in_doc || key > T);
      }
    }
    for (int o = 16; o > 0; o >>= 1) {
      ceq += __shfl_xor_sync(full, ceq, o);
      cbase += __shfl_xor_sync(full, cbase, o);
    }
    if (lane == 0) {
      S.warp_tot[warp] = ceq;
      S.warp_base[warp] = cbase;
    }
    __syncthreads();
    if (warp == 0) {   // this CTA's two counts, published to the peers
      uint32_t te = lane < kWarps ? S.warp_tot[lane] : 0u;
      uint32_t tb = lane < kWarps ? S.warp_base[lane] : 0u;
      for (int o = 16; o > 0; o >>= 1) {
        te += __shfl_xor_sync(full, te, o);
        tb += __shfl_xor_sync(full, tb, o);
      }
      if (lane == 0) {
        S.cta_eq = te;
        S.cta_keep = tb;
      }
    }
    cluster.sync();
    if (warp == 0) {
      // Ties kept before a point = min(need, ties before it): from every CTA's and
      // every warp's (tie, tie-independent) counts, exclusive scans in rank and warp
      // order give each CTA's and warp's output offset. Lane r reads peer r.
      const bool peer = lane < static_cast<int>(csize);
      const uint32_t er = peer ? *cluster.map_shared_rank(&S.cta_eq, lane) : 0u;
      const uint32_t br = peer ? *cluster.map_shared_rank(&S.cta_keep, lane) : 0u;
      __syncwarp();   // reconverge before the shuffles (without it this block took ~3 us)
      const uint32_t eq_before = warp_incl_scan(er, lane) - er;
      const uint32_t kr = br + (need > eq_before ? min(need - eq_before, er) : 0u);
      const uint32_t kr_incl = warp_incl_scan(kr, lane);
      const uint32_t keep_total = __shfl_sync(full, kr_incl, 31);
      const uint32_t cta_eq_off = __shfl_sync(full, eq_before, rank);
      const uint32_t cta_keep_off = __shfl_sync(full, kr_incl - kr, rank);
      const uint32_t ew = lane < kWarps ? S.warp_tot[lane] : 0u;
      const uint32_t bw = lane < kWarps ? S.warp_base[lane] : 0u;
      const uint32_t e_off = cta_eq_off + warp_incl_scan(ew, lane) - ew;
      const uint32_t kw = bw + (need > e_off ? min(need - e_off, ew) : 0u);
      const uint32_t k_off = cta_keep_off + warp_incl_scan(kw, lane) - kw;
      if (lane < kWarps) {
        S.warp_eq_off[lane] = e_off;
        S.warp_off[lane] = k_off;
      }
      if (lane == 0) S.seq_keep = keep_total;
    }
    __syncthreads();
    // this CTA reads no peer's shared memory after this point: announce it now and
    // wait for the peers only before exiting, so the barrier overlaps pass 2
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  }

  // ---- pass 2: keep decisions and output, ascending ----
  const int64_t seq_keep = S.seq_keep;
  const int64_t expect = len - nd + k_eff;
  const bool ok = seq_keep == expect && out_base + seq_keep <= total_kept;
  if (ok) {
    uint32_t run_eq = S.warp_eq_off[warp];
    int64_t run_out = out_base + S.warp_off[warp];
    for (int st = 0; st < nsteps; ++st) {
      const uint4 kk = k4[st * 32 + lane];
      const int i4 = seg0 + st * 128 + lane * 4;
      // per lane: ties (document keys == T) and tokens kept regardless of ties;
      // one scan of both counts packed in 16-bit halves (each total <= 128)
      uint32_t ce = 0, cb = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = i4 + e;
        const bool in_doc = i >= ld0 && i < ld1;
        const uint32_t key = key_at(kk, e);
        ce += in_doc && key == T;
        cb += i < n_local && (!in_doc || key > T);
      }
      const uint32_t packed = (ce << 16) | cb;
      const uint32_t incl = warp_incl_scan(packed, lane);
      const uint32_t tot = __shfl_sync(full, incl, 31);
      const uint32_t ex_e = (incl >> 16) - ce, ex_b = (incl & 0xFFFFu) - cb;
      // ties are kept in position order while fewer than `need` have been kept
      uint32_t rk = run_eq + ex_e;
      int64_t o = run_out + ex_b + (min(need, rk) - min(need, run_eq));
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = i4 + e;
        const bool in_doc = i >= ld0 && i < ld1;
        const uint32_t key = key_at(kk, e);
        const bool eq = in_doc && key == T;
        const bool keep = i < n_local && (!in_doc || key > T || (eq && rk < need));
        rk += eq;
        if (keep && tg::in_bounds(o, total_kept, status)) {
          kept_idx[o] = (int32_t)(base + c0 + i);
          if (kept_scores) kept_scores[o] = raw[i];
          if (kept_pos) kept_pos[o] = (int32_t)(c0 + i);
          ++o;
        }
      }
      const uint32_t te = tot >> 16, tb = tot & 0xFFFFu;
      run_out += tb + (min(need, run_eq + te) - min(need, run_eq));
      run_eq += te;
    }
  }
  if (!ok) {
    reject(out_base, expect);
  } else if (rank == 0 && tid == 0) {
    if (b == 0) cu_kept[0] = 0;
    cu_kept[b + 1] = (int32_t)(out_base + expect);
    if (b == batch - 1 && out_base + expect != total_kept) tg::set_status(status, TG_ERR_DEVICE_CHECK);
  }
  // peers may read this CTA's shared memory until they have arrived above
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// The largest cluster this device runs for the kernel: 16 CTAs (non-portable) when a
// 16-CTA cluster with the largest shared-memory footprint it would use can be
// resident, else the portable 8. Probed once per device; 0 if the runtime fails.
int max_cluster_here() {
  constexpr int kDevices = 64;
  static int cache[kDevices];   // 0: not probed yet
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kDevices) return 0;
  std::lock_guard<std::mutex> lk(mu);
  if (cache[dev] == 0) {
    int best = kPortableCluster;
    const int chunk16 = select_chunk(TG_SELECT_MAX_SEQLEN, kMaxCluster);
    const size_t smem16 = sizeof(SelectSmem) + (size_t)chunk16 * 8;
    if (cudaFuncSetAttribute(select_topk_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed,
                             1) == cudaSuccess &&
        tg::ensure_smem(reinterpret_cast<const void*>(select_topk_kernel), (int)smem16)) {
      cudaLaunchConfig_t cfg = {};
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = kMaxCluster;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.gridDim = dim3(kMaxCluster, 1, 1);
      cfg.blockDim = dim3(kThreads, 1, 1);
      cfg.dynamicSmemBytes = smem16;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int clusters = 0;
      if (cudaOccupancyMaxActiveClusters(&clusters, select_topk_kernel, &cfg) == cudaSuccess &&
          clusters > 0)
        best = kMaxCluster;
    }
    (void)cudaGetLastError();   // a refused probe leaves no error behind
    cache[dev] = best;
  }
  return cache[dev];
}

}  // namespace

extern "C" tg_status tg_select_topk(const float* scores, const int32_t* cu_seqlens,
                                    const int32_t* doc_begin, const int32_t* doc_end,
                                    const int32_t* k_doc, int batch, int64_t total_tokens,
                                    int64_t total_kept, int max_seqlen, int32_t* kept_idx,
                                    float* kept_scores, int32_t* kept_pos, int32_t* cu_kept,
                                    tg_stream_t stream) {
  tg::NvtxRange nvtx_range("tg_select_topk");
  if (batch < 0 || total_tokens < 0 || total_kept < 0 || max_seqlen < 0) return TG_ERR_INVALID_ARG;
  if (batch == 0) return TG_OK;
  if (!cu_seqlens || !doc_begin || !doc_end || !k_doc || !cu_kept) return TG_ERR_INVALID_ARG;
  if (total_tokens > 0 && !scores) return TG_ERR_INVALID_ARG;
  if (total_kept > 0 && !kept_idx) return TG_ERR_INVALID_ARG;
  if (total_kept > total_tokens || total_tokens > INT32_MAX) return TG_ERR_INVALID_ARG;
  if (max_seqlen > TG_SELECT_MAX_SEQLEN) return TG_ERR_UNSUPPORTED;
  if (batch > 65535) return TG_ERR_UNSUPPORTED;
  int* st = tg::status_word();
  if (!st) return TG_ERR_CUDA;
  const int csize = select_cluster(max_seqlen, max_cluster_here());
  if (csize <= 0) return TG_ERR_CUDA;
  const int chunk = select_chunk(max_seqlen, csize);
  if (chunk > kMaxKeysPerCta) return TG_ERR_UNSUPPORTED;
  const size_t smem = sizeof(SelectSmem) + (size_t)chunk * 8;
  if (!tg::ensure_smem(reinterpret_cast<const void*>(select_topk_kernel), (int)smem))
    return TG_ERR_CUDA;
  return tg::launch(select_topk_kernel, dim3(csize, batch, 1), dim3(kThreads), smem, stream, csize,
                    scores, cu_seqlens, doc_begin, doc_end, k_doc, batch, total_tokens,
                    total_kept, chunk,
                    kept_idx, kept_scores, kept_pos, cu_kept, st);
}

// tg_compact_kv: stable compaction of kept rows (MarkTechPost page on TokenGate,
// section "Comment TokenGate a-t-il appris le fonctionnement de la réduction des
// tokens ?": layers above the gate layer process only the K kept tokens).
//
// dst[t][r] = src[t][kept_idx[r]] for up to 8 tensors at once (an index outside
// [0, n_src_rows) is skipped and recorded as a device-check error). One warp moves one
// row of every tensor; each lane issues 128-bit non-allocating loads, eight in
// flight before the matching stores, so a 4 KB hidden-state row is one batch of 8
// fully coalesced 512-byte warp transactions. Pure HBM traffic: 2 * K * row_bytes.
#include "common.cuh"

namespace {

constexpr int kMaxTensors = 8;
constexpr int kThreads = 256;

struct CompactArgs {
  const uint4* src[kMaxTensors];
  uint4* dst[kMaxTensors];
  int64_t vecs[kMaxTensors];   // 16-byte vectors per row
  int n;
};

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__global__ void __launch_bounds__(kThreads) compact_rows_kernel(CompactArgs a,
                                                                const int32_t* __restrict__ idx,
                                                                int64_t n_kept, int64_t n_src,
                                                                int* status) {
  tg::pdl_launch_dependents();
  tg::pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kThreads) >> 5;
  for (int64_t r = warp; r < n_kept; r += nwarps) {
    const int64_t sr = idx[r];
    if (sr < 0 || sr >= n_src) {   // not a row of the sources: skip it, record the error
      if (lane == 0) tg::set_status(status, TG_ERR_DEVICE_CHECK);
      continue;
    }
    for (int t = 0; t < a.n; ++t) {
      const int64_t nv = a.vecs[t];
      const uint4* s = a.src[t] + sr * nv;
      uint4* d = a.dst[t] + r * nv;
      int64_t v = lane;
      for (; v + 224 < nv; v += 256) {   // 8 loads in flight per lane before the stores
        uint4 x[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
          x[u] = tg::in_bounds(sr * nv + v + 32 * u, n_src * nv, status) ? ld_stream(s + v + 32 * u)
                                                                          : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (tg::in_bounds(r * nv + v + 32 * u, n_kept * nv, status)) d[v + 32 * u] = x[u];
      }
      for (; v < nv; v += 32)
        if (tg::in_bounds(sr * nv + v, n_src * nv, status) &&
            tg::in_bounds(r * nv + v, n_kept * nv, status))
          d[v] = ld_stream(s + v);
    }
  }
}

}  // namespace

extern "C" tg_status tg_compact_kv(const void* const* src, void* const* dst,
                                   const int64_t* row_bytes, int n_tensors,
                                   const int32_t* kept_idx, int64_t n_kept, int64_t n_src_rows,
                                   tg_stream_t stream) {
  tg::NvtxRange nvtx_range("tg_compact_kv");
  if (!src || !dst || !row_bytes || n_tensors < 1 || n_tensors > kMaxTensors || n_kept < 0 ||
      n_src_rows < 0)
    return TG_ERR_INVALID_ARG;
  if (n_kept == 0) return TG_OK;
  if (!kept_idx) return TG_ERR_INVALID_ARG;
  CompactArgs a{};
  a.n = n_tensors;
  for (int t = 0; t < n_tensors; ++t) {
    if (!src[t] || !dst[t] || row_bytes[t] <= 0) return TG_ERR_INVALID_ARG;
    if ((row_bytes[t] & 15) || !tg::aligned16(src[t]) || !tg::aligned16(dst[t]))
      return TG_ERR_MISALIGNED;
    a.src[t] = static_cast<const uint4*>(src[t]);
    a.dst[t] = static_cast<uint4*>(dst[t]);
    a.vecs[t] = row_bytes[t] / 16;
  }
  int* st = tg::status_word();
  if (!st) return TG_ERR_CUDA;
  const int64_t warps_needed = n_kept;
  int64_t blocks = (warps_needed + (kThreads / 32) - 1) / (kThreads / 32);
  if (blocks > 148 * 16) blocks = 148 * 16;
  return tg::launch(compact_rows_kernel, dim3(static_cast<unsigned>(blocks)), dim3(kThreads), 0,
                    stream, 0, a, kept_idx, n_kept, n_src_rows, st);
}

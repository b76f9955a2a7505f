// Pieces of expert parallelism ("MoE Training: Mixture of Experts" page, Core Concepts 4, "Expert
// Parallelism": experts placed on different workers, each token's rows sent to the worker that holds
// its expert and the results sent back):
//
//   moe_copy_row_segments   row copies between any device buffers, described by a segment table in
//                           device memory.  One launch moves every segment a worker receives (the
//                           dispatch) or sends back (the return).  The source and destination of a
//                           segment are plain device pointers, so the same kernel pulls from another
//                           GPU's buffer when that buffer is peer-mapped: remote rows land in local
//                           memory before any TMA load of the GEMMs reads them.
//   moe_expert_ffn_rows     the grouped expert FFN over caller-given rows, grouped by expert: the
//                           computation a worker runs on the rows it received for its own experts.
#include <stdint.h>

#include <nvtx3/nvToolsExt.h>

#include "moe_internal.cuh"

namespace moe {
namespace {

// One grid row (blockIdx.y) per segment; the blocks of that row copy its rows in 16-byte vectors,
// four loads in flight per thread.  A segment whose pointers are not 16-byte aligned is skipped and
// recorded in the optional error word.
__global__ void __launch_bounds__(256) copy_segments_kernel(const moe_row_segment_t* __restrict__ segs,
                                                            long long vec_per_row, int32_t* status) {
  const moe_row_segment_t sg = segs[blockIdx.y];
  if (sg.rows <= 0) return;
  if (((reinterpret_cast<uintptr_t>(sg.src) | reinterpret_cast<uintptr_t>(sg.dst)) & 15u) != 0) {
    if (status && threadIdx.x == 0 && blockIdx.x == 0) atomicCAS(status, 0, kDevBadIndex);
    return;
  }
  const uint4* s = reinterpret_cast<const uint4*>(sg.src);
  uint4* d = reinterpret_cast<uint4*>(sg.dst);
  const long long n = (long long)sg.rows * vec_per_row;
  constexpr int U = 4;
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long i0 = (long long)blockIdx.x * blockDim.x + threadIdx.x; i0 < n; i0 += stride * U) {
    uint4 v[U];
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (i0 + u * stride < n) v[u] = s[i0 + u * stride];
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (i0 + u * stride < n) d[i0 + u * stride] = v[u];
  }
}

// The caller's expert offsets, made safe to index with: clamped to [0, rows_cap] and made
// non-decreasing.  Any change is recorded in the error word (results are then not meaningful).
__global__ void sanitize_offsets_kernel(const int32_t* __restrict__ in, int E, long long rows_cap, int32_t* out,
                                        int32_t* status) {
  if (threadIdx.x != 0) return;
  long long prev = 0;
  bool bad = false;
  for (int e = 0; e <= E; ++e) {
    long long v = in[e];
    if (e == 0 && v != 0) bad = true;
    if (v < prev) {
      v = prev;
      bad = true;
    }
    if (v > rows_cap) {
      v = rows_cap;
      bad = true;
    }
    out[e] = e == 0 ? 0 : (int32_t)v;
    prev = e == 0 ? 0 : v;
  }
  if (bad) atomicCAS(status, 0, kDevBadIndex);
}

size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

// Workspace of moe_expert_ffn_rows: [error word, 256 B][offsets copy (E+1) int32][h rows_cap x F].
struct RowsWs {
  size_t offsets, h, total;
};
RowsWs rows_ws(const moe_shape_t& s, long long rows_cap) {
  RowsWs w{};
  const size_t es = s.dtype == MOE_DTYPE_BF16 ? 2 : 4;
  w.offsets = 256;
  w.h = align256(w.offsets + ((size_t)s.E + 1) * 4);
  w.total = align256(w.h + (size_t)rows_cap * (size_t)s.F * es);
  return w;
}

moe_status_t check_rows_shape(const moe_shape_t* s, long long rows_cap) {
  if (s == nullptr) return MOE_ERR_INVALID_ARG;
  if (s->H <= 0 || s->E <= 0 || s->F <= 0 || s->E > 256 || rows_cap < 0) return MOE_ERR_INVALID_ARG;
  if (s->dtype != MOE_DTYPE_F32 && s->dtype != MOE_DTYPE_BF16) return MOE_ERR_INVALID_ARG;
  if (s->activation != MOE_ACT_GELU && s->activation != MOE_ACT_SILU) return MOE_ERR_INVALID_ARG;
  if (s->dtype == MOE_DTYPE_BF16 && (s->H % 64 != 0 || s->F % 64 != 0)) return MOE_ERR_UNSUPPORTED;
  if (s->dtype == MOE_DTYPE_F32 && (s->H % 4 != 0 || s->F % 4 != 0)) return MOE_ERR_UNSUPPORTED;
  const long long widest = s->H > s->F ? s->H : s->F;
  if (rows_cap * widest >= (1LL << 31)) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int device_sms() {
  static const int n = [] {
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        v <= 0)
      v = 148;
    return v;
  }();
  return n;
}

}  // namespace
}  // namespace moe

extern "C" {

moe_status_t moe_copy_row_segments(const moe_row_segment_t* segs, int nsegs, int64_t row_bytes, int64_t max_rows,
                                   int32_t* status, cudaStream_t stream) {
  moe::NvtxRange nvtx_range("moe_copy_row_segments");
  int& launches = moe::launch_count();
  launches = 0;
  if (nsegs < 0 || nsegs > 65535 || row_bytes <= 0 || row_bytes % 16 != 0 || max_rows < 0) return MOE_ERR_INVALID_ARG;
  if (nsegs == 0 || max_rows == 0) return MOE_OK;
  if (segs == nullptr || !moe::aligned16(segs)) return MOE_ERR_INVALID_ARG;
  const long long vpr = row_bytes / 16;
  long long want = (max_rows * vpr + 256 * 4 - 1) / (256 * 4);  // blocks for the longest segment
  const long long cap = 4LL * moe::device_sms();
  if (want > cap) want = cap;
  if (want < 1) want = 1;
  ++launches;
  moe::copy_segments_kernel<<<dim3((unsigned)want, (unsigned)nsegs), 256, 0, stream>>>(segs, vpr, status);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

size_t moe_expert_ffn_rows_workspace_size(const moe_shape_t* shape, int64_t rows_cap) {
  if (moe::check_rows_shape(shape, rows_cap) != MOE_OK) return 0;
  return moe::rows_ws(*shape, rows_cap).total;
}

moe_status_t moe_expert_ffn_rows(const moe_shape_t* shape, int64_t rows_cap, const int32_t* offsets, const void* x_rows,
                                 const void* W1, const void* b1, const void* W2, const void* b2, float* y, void* ws,
                                 size_t ws_bytes, cudaStream_t stream) {
  moe::NvtxRange nvtx_range("moe_expert_ffn_rows");
  int& launches = moe::launch_count();
  launches = 0;
  moe_status_t st = moe::check_rows_shape(shape, rows_cap);
  if (st != MOE_OK) return st;
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MOE_ERR_INVALID_ARG;
  const moe::RowsWs L = moe::rows_ws(*shape, rows_cap);
  if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
  if (rows_cap == 0) return MOE_OK;
  if (offsets == nullptr || x_rows == nullptr || W1 == nullptr || W2 == nullptr || y == nullptr)
    return MOE_ERR_INVALID_ARG;
  if (!moe::aligned16(x_rows) || !moe::aligned16(W1) || !moe::aligned16(W2) || !moe::aligned16(y) ||
      !moe::aligned16(b1) || !moe::aligned16(b2))
    return MOE_ERR_INVALID_ARG;
  uint8_t* base = static_cast<uint8_t*>(ws);
  int32_t* status = reinterpret_cast<int32_t*>(base);
  int32_t* offs = reinterpret_cast<int32_t*>(base + L.offsets);
  ++launches;
  moe::sanitize_offsets_kernel<<<1, 32, 0, stream>>>(offsets, shape->E, rows_cap, offs, status);
  if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  moe::FfnArgs a{};
  a.T = (int)rows_cap;
  a.H = shape->H;
  a.E = shape->E;
  a.F = shape->F;
  a.k = 1;
  a.rows_cap = (int)rows_cap;
  a.avg_rows = rows_cap / shape->E;
  a.offsets = offs;
  a.x_perm = x_rows;
  a.W1 = W1;
  a.b1 = b1;
  a.W2 = W2;
  a.b2 = b2;
  a.act = shape->activation;
  a.h = base + L.h;
  a.y = y;
  a.fuse_combine = 0;
  a.status = status;
  a.wait_limit = moe::wait_limit();
  a.num_sms = moe::device_sms();
  cudaError_t err = shape->dtype == MOE_DTYPE_BF16 ? moe::launch_ffn_bf16_sm100(a, stream, &launches)
                                                   : moe::launch_ffn_f32(a, stream, &launches);
  return err == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // extern "C"

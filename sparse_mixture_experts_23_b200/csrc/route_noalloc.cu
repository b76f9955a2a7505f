// moe_route_noalloc: the router stage for callers that cannot allocate device memory.
//
// Some callers cannot hand this library a workspace: code that runs inside another runtime's
// fixed device-memory pool with no room to carve from, latency-critical serving paths where any
// device allocation is forbidden once the process is up, and plugins whose host framework owns
// every allocation.  For them this entry point runs the same router kernels as moe_route, but
// keeps the router's scratch (per-block softmax sums, lse^2 sums and per-chunk expert
// histograms) in a fixed array compiled into the library instead of in a caller workspace.
//
// The array is a file-scope __device__ object, so every GPU that loads the library holds it
// until the process exits.  Host code must not use the array's name as a device address: it only
// names a host-side stand-in.  The device address comes from cudaGetSymbolAddress with the device
// current and is handed to the kernels as a plain pointer.  It is looked up again on every call
// made outside stream capture, so a context torn down and rebuilt (cudaDeviceReset) gets the
// array's new address; a call made while its stream is capturing uses the address of the last
// uncaptured call on that device, and fails if there was none.
#include <mutex>

#include "moe_internal.cuh"

namespace {

constexpr size_t kScratchBytes = 1u << 20;  // 1 MiB
__device__ __align__(256) unsigned char g_route_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of g_route_scratch on the current device: looked up now when `stream` is not
// capturing (and remembered for the device), else the remembered one.
cudaError_t scratch_for_current_device(cudaStream_t stream, void** out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  err = cudaStreamIsCapturing(stream, &cap);
  if (err != cudaSuccess) return err;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (cap == cudaStreamCaptureStatusNone) {
    void* p = nullptr;
    err = cudaGetSymbolAddress(&p, g_route_scratch);
    if (err != cudaSuccess) return err;
    g_scratch_ptr[dev] = p;
  } else if (g_scratch_ptr[dev] == nullptr) {
    return cudaErrorStreamCaptureUnsupported;  // no uncaptured call on this device yet
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

// Scratch layout for a shape: a device error word (256 bytes; the tensor-core gate's bounded waits
// record a timeout there), router partials [nblk][E+1] fp32, chunk histograms [k][nblk][E] int32,
// per-expert totals [E] int32, each section 256-byte aligned.
constexpr size_t kStatusBytes = 256;
size_t scratch_bytes(const moe_shape_t* s, size_t* part_off, size_t* hist_off, size_t* cnt_off) {
  const size_t nblk = ((size_t)s->T + moe::kChunk - 1) / moe::kChunk;
  const size_t part = align256(nblk * ((size_t)s->E + 1) * 4);
  const size_t hist = align256((size_t)s->k * nblk * (size_t)s->E * 4);
  *part_off = kStatusBytes;
  *hist_off = kStatusBytes + part;
  *cnt_off = kStatusBytes + part + hist;
  return kStatusBytes + part + hist + align256((size_t)s->E * 4);
}

int device_sms() {
  int dev = 0, v = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      v <= 0)
    v = 148;
  return v;
}

}  // namespace

extern "C" {

moe_status_t moe_route_noalloc(const moe_shape_t* shape, const moe_io_t* io, cudaStream_t stream) {
  moe::NvtxRange nvtx_range("moe_route_noalloc");
  int& launches = moe::launch_count();
  launches = 0;
  moe_status_t st = moe::check_shape(shape);  // the same argument rules as moe_route
  if (st != MOE_OK) return st;
  if (io == nullptr) return MOE_ERR_INVALID_ARG;
  if (shape->routing != MOE_ROUTING_TOKEN_CHOICE) return MOE_ERR_UNSUPPORTED;  // the selection needs a workspace
  if (io->aux_loss == nullptr || io->z_loss == nullptr) return MOE_ERR_INVALID_ARG;
  size_t part_off = 0, hist_off = 0, cnt_off = 0;
  if (scratch_bytes(shape, &part_off, &hist_off, &cnt_off) > kScratchBytes)
    return MOE_ERR_WORKSPACE;  // shape too large for the built-in scratch
  if (shape->T == 0) {
    ++launches;
    return moe::launch_zero_outputs(nullptr, 0, io->aux_loss, io->z_loss, stream) == cudaSuccess ? MOE_OK
                                                                                                  : MOE_ERR_CUDA;
  }
  if (io->x == nullptr || io->Wg == nullptr || io->topk_idx == nullptr || io->topk_w == nullptr)
    return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(io->x) & 15u) || (reinterpret_cast<uintptr_t>(io->Wg) & 15u))
    return MOE_ERR_INVALID_ARG;

  void* base = nullptr;
  if (scratch_for_current_device(stream, &base) != cudaSuccess) return MOE_ERR_CUDA;
  const int nblk = (shape->T + moe::kChunk - 1) / moe::kChunk;
  int32_t* status = static_cast<int32_t*>(base);
  float* loss_part = reinterpret_cast<float*>(static_cast<unsigned char*>(base) + part_off);
  int32_t* chunk_hist = reinterpret_cast<int32_t*>(static_cast<unsigned char*>(base) + hist_off);
  int32_t* cnt_pre = reinterpret_cast<int32_t*>(static_cast<unsigned char*>(base) + cnt_off);
  // Every element the kernels read from the scratch is written earlier in the same call (each
  // router block writes its whole partial row and histogram rows; the reduction writes the
  // per-expert totals before reading them), so nothing needs clearing between calls.  The error
  // word is only ever written (on a timeout), never read by a kernel; the finished-block counter
  // beside it starts at 0 (static device memory) and every call leaves it at 0.
  moe::RouterArgs r{};
  r.x = io->x;
  r.Wg = io->Wg;
  r.bg = io->bg;
  r.T = shape->T;
  r.H = shape->H;
  r.E = shape->E;
  r.k = shape->k;
  r.topk_idx = io->topk_idx;
  r.topk_w = io->topk_w;
  r.loss_part = loss_part;
  r.chunk_hist = chunk_hist;
  r.status = status;  // a bounded wait of the tensor-core gate records a timeout here
  r.wait_limit = moe::wait_limit();
  r.num_sms = device_sms();
  moe::ReduceArgs a{};
  a.T = shape->T;
  a.E = shape->E;
  a.k = shape->k;
  a.nblk = nblk;
  a.cap = -1;
  a.loss_part = loss_part;
  a.chunk_hist = chunk_hist;
  a.chunk_base = nullptr;
  a.cnt_pre = cnt_pre;
  a.expert_counts = nullptr;
  a.offsets = nullptr;
  a.aux_loss = io->aux_loss;
  a.z_loss = io->z_loss;
  a.do_losses = 1;
  a.do_dispatch = 0;
  // the losses are reduced by the router's last block (its counter sits next to the error word and
  // is back at 0 after every call), or by one reduce launch after the one-GEMM gate of 64 / 128 / 256
  // experts, which keeps its softmax / top-k tail in the GEMM epilogue.  No [T,E] gate scratch here.
  r.red = a;
  r.done = reinterpret_cast<unsigned*>(static_cast<unsigned char*>(base) + moe::kRouterDoneOffset);
  bool reduced = false;
  if (moe::launch_router(r, shape->dtype, stream, &launches, &reduced) != cudaSuccess) return MOE_ERR_CUDA;
  if (reduced) return MOE_OK;
  ++launches;
  return moe::launch_reduce(a, stream) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // extern "C"

// Host side of the C ABI declared in include/moe.h: argument validation, workspace layout and
// the launch sequence of each stage on the caller's stream.  No allocation, no synchronisation
// (except moe_get_device_status).
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <atomic>
#include <mutex>
#include <vector>

#include <nvtx3/nvToolsExt.h>  // header-only; the calls cost nothing unless a profiler is attached

#include "moe_internal.cuh"

namespace moe {

static size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

cudaError_t ensure_smem_limit(const void* kernel, int bytes) {
  struct Entry {
    const void* kernel;
    int device;
    int bytes;
  };
  static std::mutex mu;
  static std::vector<Entry> done;
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  std::lock_guard<std::mutex> lock(mu);
  for (Entry& en : done)
    if (en.kernel == kernel && en.device == dev) {
      if (en.bytes >= bytes) return cudaSuccess;
      err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
      if (err == cudaSuccess) en.bytes = bytes;
      return err;
    }
  err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (err == cudaSuccess) done.push_back({kernel, dev, bytes});
  return err;
}

// Tokens per expert under expert choice: min(T, ceil(CF*T*k/E)), T when CF = +inf.
long long ec_capacity(const moe_shape_t& s) {
  if (isinf(s.capacity_factor)) return s.T;
  double c = ceil(s.capacity_factor * (double)s.T * (double)s.k / (double)s.E);
  if (c < (double)s.min_capacity) c = (double)s.min_capacity;
  return c < (double)s.T ? (long long)c : (long long)s.T;
}

WsLayout ws_layout(const moe_shape_t& s) {
  WsLayout L{};
  const size_t T = (size_t)s.T, E = (size_t)s.E, k = (size_t)s.k;
  const size_t es = s.dtype == MOE_DTYPE_BF16 ? 2 : 4;
  const bool ec = s.routing == MOE_ROUTING_EXPERT_CHOICE;
  L.nblk = (int)((T + kChunk - 1) / kChunk);
  const size_t nblk = (size_t)L.nblk;
  L.ec_cap = ec ? (int)ec_capacity(s) : 0;
  const size_t rows = ec ? E * (size_t)L.ec_cap : T * k;
  L.rows = (long long)rows;
  size_t o = 0;
  L.status = o;
  o = align256(o + 16);
  L.offsets = o;
  o = align256(o + (E + 1) * 4);
  L.cnt_pre = o;
  o = align256(o + E * 4);
  L.chunk_hist = o;
  o = align256(o + k * nblk * E * 4);
  L.chunk_base = o;
  o = align256(o + k * nblk * E * 4);
  L.loss_part = o;
  o = align256(o + nblk * (E + 1) * 4);
  L.row_of = o;
  o = align256(o + rows * 4);
  L.row_token = o;
  o = align256(o + rows * 4);
  L.row_slot = o;
  o = align256(o + rows * 4);
  L.x_perm = o;
  o = align256(o + rows * (size_t)s.H * es);
  L.h = o;
  o = align256(o + rows * (size_t)s.F * es);
  L.y = o;
  o = align256(o + rows * (size_t)s.H * 4);
  L.scores = o;  // expert choice: [E][T] fp32 logits, then [T] per-token expert counts
  o = align256(o + (ec ? E * T * 4 : 0));
  L.tok_count = o;
  o = align256(o + (ec ? T * 4 : 0));
  L.logits = o;  // [T,E] fp32: gate logits (the tensor-core gate's output; saved for the backward pass)
  o = align256(o + T * E * 4);
  L.red_scratch = o;  // the multi-block reduction's per-expert terms (fp64) and per-block z partials
  o = align256(o + 256 * 8 + 256 * 4);
  L.total = o;
  // training sections (moe_forward_train / moe_backward), appended after the inference layout
  L.u = o;
  o = align256(o + rows * (size_t)s.F * es);
  L.dperm = o;
  o = align256(o + rows * (size_t)s.H * es);
  L.dyperm = o;
  o = align256(o + rows * (size_t)s.H * es);
  L.du = o;
  o = align256(o + rows * (size_t)s.F * es);
  L.dwraw = o;
  o = align256(o + rows * 4);
  L.dlogits = o;
  o = align256(o + T * E * 4);
  L.train_total = o;
  return L;
}

}  // namespace moe

using namespace moe;

namespace {

thread_local int g_launches = 0;

// bound on device-side waits for launches made after moe_set_wait_limit (any host thread may set it)
std::atomic<long long> g_wait_limit{2000000000LL};
// kernel-selection flags of moe_set_kernel_options (any host thread may set them)
std::atomic<int> g_kernel_options{0};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

namespace moe {

int& launch_count() { return g_launches; }
int kernel_options() { return g_kernel_options.load(std::memory_order_relaxed); }
long long wait_limit() { return g_wait_limit.load(); }

// One NVTX range per entry-point call ("moe_route", "moe_forward", ...), so that a timeline shows the
// stages of a layer call around its kernels.
NvtxRange::NvtxRange(const char* name) { nvtxRangePushA(name); }
NvtxRange::~NvtxRange() { nvtxRangePop(); }

moe_status_t check_shape(const moe_shape_t* s) {
  if (s == nullptr) return MOE_ERR_INVALID_ARG;
  if (s->T < 0 || s->H <= 0 || s->E <= 0 || s->F <= 0 || s->k <= 0) return MOE_ERR_INVALID_ARG;
  if (s->k > s->E || s->k > 8 || s->E > 256) return MOE_ERR_INVALID_ARG;
  if (!(s->capacity_factor > 0.0)) return MOE_ERR_INVALID_ARG;  // also rejects NaN
  if (s->dtype != MOE_DTYPE_F32 && s->dtype != MOE_DTYPE_BF16) return MOE_ERR_INVALID_ARG;
  if (s->activation != MOE_ACT_GELU && s->activation != MOE_ACT_SILU) return MOE_ERR_INVALID_ARG;
  if (s->routing != MOE_ROUTING_TOKEN_CHOICE && s->routing != MOE_ROUTING_EXPERT_CHOICE) return MOE_ERR_INVALID_ARG;
  if (s->min_capacity < 0) return MOE_ERR_INVALID_ARG;
  if (s->dtype == MOE_DTYPE_BF16 && (s->H % 64 != 0 || s->F % 64 != 0)) return MOE_ERR_UNSUPPORTED;
  if (s->dtype == MOE_DTYPE_F32 && (s->H % 4 != 0 || s->F % 4 != 0)) return MOE_ERR_UNSUPPORTED;
  const long long rows =
      s->routing == MOE_ROUTING_EXPERT_CHOICE ? (long long)s->E * ec_capacity(*s) : (long long)s->T * s->k;
  const long long widest = s->H > s->F ? s->H : s->F;
  if (rows * widest >= (1LL << 31)) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

}  // namespace moe

namespace {

long long capacity_of(const moe_shape_t* s) {
  if (isinf(s->capacity_factor)) return -1;
  double c = ceil(s->capacity_factor * (double)s->T * (double)s->k / (double)s->E);
  if (c < (double)s->min_capacity) c = (double)s->min_capacity;
  if (c >= (double)((long long)s->T * s->k)) return -1;  // never binding
  return (long long)c;
}

moe_status_t check_ws(const moe_shape_t* s, const void* ws, size_t ws_bytes) {
  if (ws == nullptr) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < ws_layout(*s).total) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

moe_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

int num_sms() {
  static const int n = [] {  // initialised once, thread-safely, on the first call
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
      v = 148;
    return v;
  }();
  return n;
}

// ---------------------------------------------------------------- stage bodies (validated) -------
ReduceArgs reduce_args(const moe_shape_t* s, const moe_io_t* io, void* ws, int do_losses, int do_dispatch);
// reduce: which reductions follow the router (kReduceLosses, kReduceDispatch; token choice only).  The
// router's last block runs them when the chosen router kernel can, else one reduce launch follows.
constexpr int kReduceLosses = 1, kReduceDispatch = 2;
moe_status_t do_route(const moe_shape_t* s, const moe_io_t* io, void* ws, cudaStream_t st, int reduce,
                      bool train = false) {
  const WsLayout L = ws_layout(*s);
  if (s->T == 0) {
    ++g_launches;
    return cuda_status(launch_zero_outputs(nullptr, 0, io->aux_loss, io->z_loss, st));
  }
  RouterArgs r{};
  r.x = io->x;
  r.Wg = io->Wg;
  r.bg = io->bg;
  r.T = s->T;
  r.H = s->H;
  r.E = s->E;
  r.k = s->k;
  r.topk_idx = io->topk_idx;
  r.topk_w = io->topk_w;
  r.loss_part = at<float>(ws, L.loss_part);
  r.chunk_hist = at<int32_t>(ws, L.chunk_hist);
  r.logits_out = train ? at<float>(ws, L.logits) : nullptr;
  if (s->routing == MOE_ROUTING_EXPERT_CHOICE) {
    r.chunk_hist = nullptr;
    r.scores = at<float>(ws, L.scores);
    r.tok_count = at<int32_t>(ws, L.tok_count);
  }
  r.gemm_logits = at<float>(ws, L.logits);
  r.status = at<int32_t>(ws, L.status);
  r.wait_limit = g_wait_limit;
  r.num_sms = num_sms();
  if (reduce != 0 && s->routing != MOE_ROUTING_EXPERT_CHOICE) {
    r.red = reduce_args(s, io, ws, (reduce & kReduceLosses) != 0, (reduce & kReduceDispatch) != 0);
    r.done = at<unsigned>(ws, L.status + kRouterDoneOffset);
  }
  bool reduced = false;
  cudaError_t err = launch_router(r, s->dtype, st, &g_launches, &reduced);
  if (err != cudaSuccess) return MOE_ERR_CUDA;
  if (r.done != nullptr && !reduced) {
    ++g_launches;
    return cuda_status(launch_reduce(r.red, st));
  }
  return MOE_OK;
}

// Expert choice, after the router: per-expert top-C selection, then the losses.
moe_status_t do_ec_select_and_losses(const moe_shape_t* s, const moe_io_t* io, void* ws, cudaStream_t st) {
  const WsLayout L = ws_layout(*s);
  EcSelectArgs a{};
  a.scores = at<float>(ws, L.scores);
  a.T = s->T;
  a.E = s->E;
  a.C = L.ec_cap;
  a.chosen = io->topk_idx;
  a.expert_counts = io->expert_counts;
  a.cnt_pre = at<int32_t>(ws, L.cnt_pre);
  a.tok_count = at<int32_t>(ws, L.tok_count);
  a.dropped = io->dropped;
  a.done = at<unsigned>(ws, L.status + kEcDoneOffset);
  ++g_launches;
  if (launch_ec_select(a, st) != cudaSuccess) return MOE_ERR_CUDA;
  ReduceArgs ra = reduce_args(s, io, ws, 1, 0);
  ra.ec_count = L.ec_cap;
  ++g_launches;
  return cuda_status(launch_reduce(ra, st));
}

moe_status_t do_ec_gather(const moe_shape_t* s, const moe_io_t* io, void* ws, cudaStream_t st, bool clear_out = true) {
  const WsLayout L = ws_layout(*s);
  EcGatherArgs a{};
  a.status = at<int32_t>(ws, L.status);
  a.x = io->x;
  a.T = s->T;
  a.H = s->H;
  a.E = s->E;
  a.C = L.ec_cap;
  a.esize = s->dtype == MOE_DTYPE_BF16 ? 2 : 4;
  a.chosen = io->topk_idx;
  a.offsets = at<int32_t>(ws, L.offsets);
  a.row_token = at<int32_t>(ws, L.row_token);
  a.row_slot = at<int32_t>(ws, L.row_slot);
  a.x_perm = at<void>(ws, L.x_perm);
  a.out = clear_out ? io->out : nullptr;
  ++g_launches;
  return cuda_status(launch_ec_gather(a, st));
}

ReduceArgs reduce_args(const moe_shape_t* s, const moe_io_t* io, void* ws, int do_losses, int do_dispatch) {
  const WsLayout L = ws_layout(*s);
  ReduceArgs a{};
  a.T = s->T;
  a.E = s->E;
  a.k = s->k;
  a.nblk = L.nblk;
  a.cap = capacity_of(s);
  a.loss_part = at<float>(ws, L.loss_part);
  a.chunk_hist = at<int32_t>(ws, L.chunk_hist);
  a.chunk_base = at<int32_t>(ws, L.chunk_base);
  a.cnt_pre = at<int32_t>(ws, L.cnt_pre);
  a.expert_counts = io->expert_counts;
  a.offsets = at<int32_t>(ws, L.offsets);
  a.aux_loss = io->aux_loss;
  a.z_loss = io->z_loss;
  a.do_losses = do_losses;
  a.do_dispatch = do_dispatch;
  a.terms = at<double>(ws, L.red_scratch);
  a.zpart = at<float>(ws, L.red_scratch + 256 * 8);
  a.done = at<unsigned>(ws, L.status + kReduceDoneOffset);
  return a;
}

moe_status_t do_scatter(const moe_shape_t* s, const moe_io_t* io, void* ws, cudaStream_t st, bool clear_out = true) {
  const WsLayout L = ws_layout(*s);
  ScatterArgs a{};
  a.status = at<int32_t>(ws, L.status);
  a.x = io->x;
  a.T = s->T;
  a.H = s->H;
  a.E = s->E;
  a.k = s->k;
  a.nblk = L.nblk;
  a.esize = s->dtype == MOE_DTYPE_BF16 ? 2 : 4;
  a.cap = capacity_of(s);
  a.topk_idx = io->topk_idx;
  a.chunk_base = at<int32_t>(ws, L.chunk_base);
  a.offsets = at<int32_t>(ws, L.offsets);
  a.dropped = io->dropped;
  a.row_of = at<int32_t>(ws, L.row_of);
  a.row_token = at<int32_t>(ws, L.row_token);
  a.row_slot = at<int32_t>(ws, L.row_slot);
  a.x_perm = at<void>(ws, L.x_perm);
  a.out = clear_out ? io->out : nullptr;
  ++g_launches;
  return cuda_status(launch_scatter(a, num_sms(), st));
}

// Expected rows per expert, for the FFN's tile-shape choice: T*k/E, or C under expert choice.
long long ffn_avg_rows(const moe_shape_t* s) {
  return s->routing == MOE_ROUTING_EXPERT_CHOICE ? ws_layout(*s).ec_cap : (long long)s->T * s->k / s->E;
}

// Whole forward: whether GEMM1 zeroes out (its CTA-pair form, whose epilogue warps are idle during
// the first tile) in place of the scatter or gather, which then only copy rows.
bool gemm1_clears_out(const moe_shape_t* s) {
  return s->dtype == MOE_DTYPE_BF16 && ffn_gemm1_on_pairs(s->H, s->F, ffn_avg_rows(s));
}

moe_status_t do_ffn(const moe_shape_t* s, const moe_io_t* io, void* ws, int fuse, cudaStream_t st, bool train = false,
                    bool clear_out = false) {
  const WsLayout L = ws_layout(*s);
  FfnArgs a{};
  a.T = s->T;
  a.H = s->H;
  a.E = s->E;
  a.F = s->F;
  a.k = s->k;
  const bool ec = s->routing == MOE_ROUTING_EXPERT_CHOICE;
  a.rows_cap = (int)L.rows;
  // under expert choice row_slot holds the expert, so the weight of row r is topk_w[t*E + e]
  if (ec) a.k = s->E;
  a.avg_rows = ffn_avg_rows(s);
  a.offsets = at<int32_t>(ws, L.offsets);
  a.row_token = at<int32_t>(ws, L.row_token);
  a.row_slot = at<int32_t>(ws, L.row_slot);
  a.topk_w = io->topk_w;
  a.x_perm = at<void>(ws, L.x_perm);
  a.W1 = io->W1;
  a.b1 = io->b1;
  a.W2 = io->W2;
  a.b2 = io->b2;
  a.h = at<void>(ws, L.h);
  a.y = at<float>(ws, L.y);
  a.out = io->out;
  a.fuse_combine = fuse;
  a.u_out = train ? at<void>(ws, L.u) : nullptr;
  a.act = s->activation;
  a.status = at<int32_t>(ws, L.status);
  a.wait_limit = g_wait_limit;
  a.num_sms = num_sms();
  a.clear_out = clear_out ? io->out : nullptr;
  cudaError_t err = s->dtype == MOE_DTYPE_BF16 ? launch_ffn_bf16_sm100(a, st, &g_launches) : launch_ffn_f32(a, st, &g_launches);
  return cuda_status(err);
}

bool null_any(std::initializer_list<const void*> ps) {
  for (const void* p : ps)
    if (p == nullptr) return true;
  return false;
}

}  // namespace

extern "C" {

size_t moe_workspace_size(const moe_shape_t* shape) {
  if (check_shape(shape) != MOE_OK) return 0;
  return ws_layout(*shape).total;
}

int64_t moe_capacity(const moe_shape_t* shape) {
  if (check_shape(shape) != MOE_OK) return -2;
  if (shape->routing == MOE_ROUTING_EXPERT_CHOICE) return ec_capacity(*shape);
  if (isinf(shape->capacity_factor)) return -1;
  const int64_t c = (int64_t)ceil(shape->capacity_factor * (double)shape->T * (double)shape->k / (double)shape->E);
  return c > shape->min_capacity ? c : (int64_t)shape->min_capacity;
}

moe_status_t moe_workspace_layout(const moe_shape_t* shape, void* ws, moe_ws_view_t* view) {
  moe_status_t st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (ws == nullptr || view == nullptr) return MOE_ERR_INVALID_ARG;
  const WsLayout L = ws_layout(*shape);
  view->status = at<int32_t>(ws, L.status);
  view->offsets = at<int32_t>(ws, L.offsets);
  view->cnt_pre = at<int32_t>(ws, L.cnt_pre);
  view->row_of = at<int32_t>(ws, L.row_of);
  view->row_token = at<int32_t>(ws, L.row_token);
  view->row_slot = at<int32_t>(ws, L.row_slot);
  view->x_perm = at<void>(ws, L.x_perm);
  view->h = at<void>(ws, L.h);
  view->y = at<float>(ws, L.y);
  view->bytes = L.total;
  view->scores = shape->routing == MOE_ROUTING_EXPERT_CHOICE ? at<float>(ws, L.scores) : nullptr;
  return MOE_OK;
}

moe_status_t moe_route(const moe_shape_t* shape, const moe_io_t* io, void* ws, size_t ws_bytes, cudaStream_t stream) {
  NvtxRange nvtx_range("moe_route");
  g_launches = 0;
  moe_status_t st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (io == nullptr) return MOE_ERR_INVALID_ARG;
  if ((st = check_ws(shape, ws, ws_bytes)) != MOE_OK) return st;
  if (null_any({io->aux_loss, io->z_loss})) return MOE_ERR_INVALID_ARG;
  const bool ec = shape->routing == MOE_ROUTING_EXPERT_CHOICE;
  if (ec && null_any({io->expert_counts})) return MOE_ERR_INVALID_ARG;
  if (shape->T == 0) {
    if (!ec) return do_route(shape, io, ws, stream, kReduceLosses);
    ++g_launches;
    return cuda_status(launch_zero_outputs(io->expert_counts, shape->E, io->aux_loss, io->z_loss, stream));
  }
  if (null_any({io->x, io->Wg, io->topk_idx, io->topk_w})) return MOE_ERR_INVALID_ARG;  // bg optional
  if (ec && null_any({io->dropped})) return MOE_ERR_INVALID_ARG;
  if (!aligned16(io->x) || !aligned16(io->Wg)) return MOE_ERR_INVALID_ARG;
  if ((st = do_route(shape, io, ws, stream, ec ? 0 : kReduceLosses)) != MOE_OK) return st;
  if (ec) return do_ec_select_and_losses(shape, io, ws, stream);
  return MOE_OK;
}

moe_status_t moe_loss_sums(const moe_shape_t* shape, void* ws, size_t ws_bytes, float* sums, cudaStream_t stream) {
  NvtxRange nvtx_range("moe_loss_sums");
  g_launches = 0;
  moe_status_t st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (sums == nullptr || (reinterpret_cast<uintptr_t>(sums) & 3u) != 0) return MOE_ERR_INVALID_ARG;
  if ((st = check_ws(shape, ws, ws_bytes)) != MOE_OK) return st;
  const WsLayout L = ws_layout(*shape);
  ++g_launches;
  return cuda_status(launch_loss_sums(at<float>(ws, L.loss_part), at<int32_t>(ws, L.cnt_pre), L.nblk, shape->E,
                                      shape->T, sums, stream));
}

moe_status_t moe_losses_from_sums(int E, const float* sums, float* aux_loss, float* z_loss, cudaStream_t stream) {
  NvtxRange nvtx_range("moe_losses_from_sums");
  g_launches = 0;
  if (E < 1 || E > 256) return MOE_ERR_INVALID_ARG;
  if (null_any({sums, aux_loss, z_loss})) return MOE_ERR_INVALID_ARG;
  ++g_launches;
  return cuda_status(launch_losses_from_sums(sums, E, aux_loss, z_loss, stream));
}

moe_status_t moe_permute(const moe_shape_t* shape, const moe_io_t* io, void* ws, size_t ws_bytes,
                         cudaStream_t stream) {
  NvtxRange nvtx_range("moe_permute");
  g_launches = 0;
  moe_status_t st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (io == nullptr) return MOE_ERR_INVALID_ARG;
  if ((st = check_ws(shape, ws, ws_bytes)) != MOE_OK) return st;
  if (null_any({io->expert_counts})) return MOE_ERR_INVALID_ARG;
  if (shape->T == 0) {
    ++g_launches;
    return cuda_status(launch_zero_outputs(io->expert_counts, shape->E, nullptr, nullptr, stream));
  }
  if (shape->routing == MOE_ROUTING_EXPERT_CHOICE) {
    if (null_any({io->x, io->topk_idx, io->out})) return MOE_ERR_INVALID_ARG;
    if (!aligned16(io->x) || !aligned16(io->out)) return MOE_ERR_INVALID_ARG;
    return do_ec_gather(shape, io, ws, stream);
  }
  if (null_any({io->x, io->topk_idx, io->dropped, io->out})) return MOE_ERR_INVALID_ARG;
  if (!aligned16(io->x) || !aligned16(io->out)) return MOE_ERR_INVALID_ARG;
  const WsLayout L = ws_layout(*shape);
  // histograms, with the dispatch reduction in the last histogram block when it fits there
  const ReduceArgs red = reduce_args(shape, io, ws, 0, 1);
  bool reduced = false;
  ++g_launches;
  if ((st = cuda_status(launch_hist(io->topk_idx, shape->T, shape->E, shape->k, L.nblk, at<int32_t>(ws, L.chunk_hist),
                                    at<int32_t>(ws, L.status), red, at<unsigned>(ws, L.status + kRouterDoneOffset),
                                    stream, &reduced))) != MOE_OK)
    return st;
  if (!reduced) {
    ++g_launches;
    if ((st = cuda_status(launch_reduce(red, stream))) != MOE_OK) return st;
  }
  return do_scatter(shape, io, ws, stream);
}

moe_status_t moe_expert_ffn(const moe_shape_t* shape, const moe_io_t* io, void* ws, size_t ws_bytes, int fuse_combine,
                            cudaStream_t stream) {
  NvtxRange nvtx_range("moe_expert_ffn");
  g_launches = 0;
  moe_status_t st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (io == nullptr) return MOE_ERR_INVALID_ARG;
  if ((st = check_ws(shape, ws, ws_bytes)) != MOE_OK) return st;
  if (shape->T == 0) return MOE_OK;
  if (null_any({io->W1, io->W2, io->topk_w})) return MOE_ERR_INVALID_ARG;  // b1, b2 optional
  if (fuse_combine && io->out == nullptr) return MOE_ERR_INVALID_ARG;
  if (!aligned16(io->W1) || !aligned16(io->W2) || !aligned16(io->b1) || !aligned16(io->b2) ||
      (fuse_combine && !aligned16(io->out)))
    return MOE_ERR_INVALID_ARG;
  return do_ffn(shape, io, ws, fuse_combine ? 1 : 0, stream);
}

moe_status_t moe_combine(const moe_shape_t* shape, const moe_io_t* io, void* ws, size_t ws_bytes, cudaStream_t stream) {
  NvtxRange nvtx_range("moe_combine");
  g_launches = 0;
  moe_status_t st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (io == nullptr) return MOE_ERR_INVALID_ARG;
  if ((st = check_ws(shape, ws, ws_bytes)) != MOE_OK) return st;
  if (shape->T == 0) return MOE_OK;
  if (null_any({io->out, io->topk_w})) return MOE_ERR_INVALID_ARG;
  if (shape->routing == MOE_ROUTING_EXPERT_CHOICE && io->topk_idx == nullptr) return MOE_ERR_INVALID_ARG;
  if (!aligned16(io->out)) return MOE_ERR_INVALID_ARG;
  const WsLayout L = ws_layout(*shape);
  ++g_launches;
  if (shape->routing == MOE_ROUTING_EXPERT_CHOICE)
    return cuda_status(launch_ec_combine(at<float>(ws, L.y), io->topk_idx, io->topk_w, shape->T, shape->E, L.ec_cap,
                                         shape->H, io->out, stream));
  return cuda_status(launch_combine(at<float>(ws, L.y), at<int32_t>(ws, L.row_of), io->topk_w, shape->T, shape->H,
                                    shape->k, io->out, stream));
}

moe_status_t moe_forward(const moe_shape_t* shape, const moe_io_t* io, void* ws, size_t ws_bytes, cudaStream_t stream) {
  NvtxRange nvtx_range("moe_forward");
  g_launches = 0;
  moe_status_t st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (io == nullptr) return MOE_ERR_INVALID_ARG;
  if ((st = check_ws(shape, ws, ws_bytes)) != MOE_OK) return st;
  if (null_any({io->aux_loss, io->z_loss, io->expert_counts})) return MOE_ERR_INVALID_ARG;
  if (shape->T == 0) {
    ++g_launches;
    return cuda_status(launch_zero_outputs(io->expert_counts, shape->E, io->aux_loss, io->z_loss, stream));
  }
  if (null_any({io->x, io->Wg, io->W1, io->W2, io->out, io->topk_idx, io->topk_w, io->dropped}))
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(io->x) || !aligned16(io->Wg) || !aligned16(io->W1) || !aligned16(io->W2) || !aligned16(io->out) ||
      !aligned16(io->b1) || !aligned16(io->b2))
    return MOE_ERR_INVALID_ARG;
  if (shape->routing == MOE_ROUTING_EXPERT_CHOICE) {
    // router, per-expert selection, losses, gather, GEMM1, GEMM2 (each call adds its launches)
    if ((st = do_route(shape, io, ws, stream, 0)) != MOE_OK) return st;
    if ((st = do_ec_select_and_losses(shape, io, ws, stream)) != MOE_OK) return st;
    const bool gc = gemm1_clears_out(shape);
    if ((st = do_ec_gather(shape, io, ws, stream, !gc)) != MOE_OK) return st;
    return do_ffn(shape, io, ws, 1, stream, false, gc);
  }
  int n = 0;
  // the router emits the chunk histograms itself, so one reduction serves losses and dispatch
  if ((st = do_route(shape, io, ws, stream, kReduceLosses | kReduceDispatch)) != MOE_OK) return st;
  n += g_launches;
  g_launches = 0;
  const bool gc = gemm1_clears_out(shape);
  if ((st = do_scatter(shape, io, ws, stream, !gc)) != MOE_OK) return st;
  n += g_launches;
  g_launches = 0;
  st = do_ffn(shape, io, ws, 1, stream, false, gc);
  g_launches += n;
  return st;
}

size_t moe_train_workspace_size(const moe_shape_t* shape) {
  if (check_shape(shape) != MOE_OK) return 0;
  return ws_layout(*shape).train_total;
}

static moe_status_t check_train(const moe_shape_t* shape, void* ws, size_t ws_bytes) {
  moe_status_t st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < ws_layout(*shape).train_total) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

moe_status_t moe_forward_train(const moe_shape_t* shape, const moe_io_t* io, void* ws, size_t ws_bytes,
                               cudaStream_t stream) {
  NvtxRange nvtx_range("moe_forward_train");
  g_launches = 0;
  moe_status_t st = check_train(shape, ws, ws_bytes);
  if (st != MOE_OK) return st;
  if (io == nullptr) return MOE_ERR_INVALID_ARG;
  if (null_any({io->aux_loss, io->z_loss, io->expert_counts})) return MOE_ERR_INVALID_ARG;
  if (shape->T == 0) {
    ++g_launches;
    return cuda_status(launch_zero_outputs(io->expert_counts, shape->E, io->aux_loss, io->z_loss, stream));
  }
  if (null_any({io->x, io->Wg, io->W1, io->W2, io->out, io->topk_idx, io->topk_w, io->dropped}))
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(io->x) || !aligned16(io->Wg) || !aligned16(io->W1) || !aligned16(io->W2) || !aligned16(io->out) ||
      !aligned16(io->b1) || !aligned16(io->b2))
    return MOE_ERR_INVALID_ARG;
  const bool ec = shape->routing == MOE_ROUTING_EXPERT_CHOICE;
  if ((st = do_route(shape, io, ws, stream, ec ? 0 : kReduceLosses | kReduceDispatch, true)) != MOE_OK) return st;
  if (ec) {
    if ((st = do_ec_select_and_losses(shape, io, ws, stream)) != MOE_OK) return st;
    const bool gc = gemm1_clears_out(shape);
    if ((st = do_ec_gather(shape, io, ws, stream, !gc)) != MOE_OK) return st;
    return do_ffn(shape, io, ws, 1, stream, true, gc);
  }
  const bool gc = gemm1_clears_out(shape);
  if ((st = do_scatter(shape, io, ws, stream, !gc)) != MOE_OK) return st;
  return do_ffn(shape, io, ws, 1, stream, true, gc);
}

moe_status_t moe_backward(const moe_shape_t* shape, const moe_io_t* io, const moe_grad_t* grad, void* ws,
                          size_t ws_bytes, cudaStream_t stream) {
  NvtxRange nvtx_range("moe_backward");
  g_launches = 0;
  moe_status_t st = check_train(shape, ws, ws_bytes);
  if (st != MOE_OK) return st;
  if (io == nullptr || grad == nullptr) return MOE_ERR_INVALID_ARG;
  if (null_any({grad->dout, grad->dx, grad->dWg, grad->dW1, grad->dW2})) return MOE_ERR_INVALID_ARG;
  // a bias gradient is wanted exactly when the layer has that bias
  if ((io->bg == nullptr) != (grad->dbg == nullptr) || (io->b1 == nullptr) != (grad->db1 == nullptr) ||
      (io->b2 == nullptr) != (grad->db2 == nullptr))
    return MOE_ERR_INVALID_ARG;
  if (shape->T == 0) return MOE_OK;
  if (null_any({io->x, io->Wg, io->W1, io->W2, io->topk_idx, io->topk_w, io->dropped})) return MOE_ERR_INVALID_ARG;
  if (!aligned16(grad->dout) || !aligned16(grad->dx) || !aligned16(io->W1) || !aligned16(io->W2))
    return MOE_ERR_INVALID_ARG;
  const WsLayout L = ws_layout(*shape);
  const bool ec = shape->routing == MOE_ROUTING_EXPERT_CHOICE;
  const int f32 = shape->dtype == MOE_DTYPE_F32 ? 1 : 0;
  const int kw = ec ? shape->E : shape->k;  // stride of the combine weights in topk_w
  const int32_t* offsets = at<int32_t>(ws, L.offsets);
  const int32_t* row_token = at<int32_t>(ws, L.row_token);
  const int32_t* row_slot = at<int32_t>(ws, L.row_slot);
  float* dlogits = at<float>(ws, L.dlogits);  // under expert choice it first holds dL/dp of the chosen pairs

  BwdPrepArgs pa{};
  pa.T = shape->T;
  pa.H = shape->H;
  pa.E = shape->E;
  pa.k = kw;
  pa.f32 = f32;
  pa.offsets = offsets;
  pa.row_token = row_token;
  pa.row_slot = row_slot;
  pa.topk_w = io->topk_w;
  pa.dout = grad->dout;
  pa.dperm = at<void>(ws, L.dperm);
  pa.dyperm = at<void>(ws, L.dyperm);
  pa.dwraw = at<float>(ws, L.dwraw);
  pa.dx = grad->dx;
  pa.dWg = grad->dWg;
  pa.dbg = grad->dbg;
  pa.F = shape->F;
  pa.db1 = grad->db1;
  pa.db2 = grad->db2;
  pa.dwmat = ec ? dlogits : nullptr;
  ++g_launches;
  if ((st = cuda_status(launch_bwd_prep(pa, stream))) != MOE_OK) return st;

  BwdGemmArgs ga{};
  ga.T = shape->T;
  ga.H = shape->H;
  ga.E = shape->E;
  ga.F = shape->F;
  ga.k = kw;
  ga.rows_cap = (int)L.rows;
  ga.act = shape->activation;
  ga.avg_rows = ec ? L.ec_cap : (long long)shape->T * shape->k / shape->E;
  ga.offsets = offsets;
  ga.row_token = row_token;
  ga.row_slot = row_slot;
  ga.topk_w = io->topk_w;
  ga.W1 = io->W1;
  ga.W2 = io->W2;
  ga.x_perm = at<void>(ws, L.x_perm);
  ga.h = at<void>(ws, L.h);
  ga.u = at<void>(ws, L.u);
  ga.dperm = pa.dperm;
  ga.dyperm = pa.dyperm;
  ga.du = at<void>(ws, L.du);
  ga.dwraw = pa.dwraw;
  ga.dx = grad->dx;
  ga.dW1 = grad->dW1;
  ga.dW2 = grad->dW2;
  ga.status = at<int32_t>(ws, L.status);
  ga.wait_limit = g_wait_limit;
  ga.num_sms = num_sms();
  if ((st = cuda_status(f32 ? launch_bwd_gemms_f32(ga, stream, &g_launches)
                            : launch_bwd_gemms_sm100(ga, stream, &g_launches))) != MOE_OK)
    return st;

  if (grad->db1 || grad->db2) {
    BiasGradArgs ba{};
    ba.H = shape->H;
    ba.F = shape->F;
    ba.E = shape->E;
    ba.k = kw;
    ba.f32 = f32;
    ba.rows_cap = (int)L.rows;
    ba.offsets = offsets;
    ba.row_token = row_token;
    ba.row_slot = row_slot;
    ba.topk_w = io->topk_w;
    ba.dout = grad->dout;
    ba.du = ga.du;
    ba.db1 = grad->db1;
    ba.db2 = grad->db2;
    ++g_launches;
    if ((st = cuda_status(launch_bias_grad(ba, stream))) != MOE_OK) return st;
  }

  if (ec) {
    EcDwArgs da{};
    da.rows = (int)L.rows;
    da.H = shape->H;
    da.E = shape->E;
    da.row_token = row_token;
    da.row_slot = row_slot;
    da.dwraw = pa.dwraw;
    da.dout = grad->dout;
    da.b2 = io->b2;
    da.f32 = f32;
    da.dwmat = dlogits;
    ++g_launches;
    if ((st = cuda_status(launch_ec_dw_scatter(da, stream))) != MOE_OK) return st;
  }

  RouterBwdArgs ra{};
  ra.T = shape->T;
  ra.H = shape->H;
  ra.E = shape->E;
  ra.k = shape->k;
  ra.logits = at<float>(ws, L.logits);
  ra.topk_idx = io->topk_idx;
  ra.topk_w = io->topk_w;
  ra.dropped = io->dropped;
  ra.row_of = at<int32_t>(ws, L.row_of);
  ra.cnt_pre = at<int32_t>(ws, L.cnt_pre);
  ra.dwraw = pa.dwraw;
  ra.dout = grad->dout;
  ra.b2 = io->b2;
  ra.Wg = io->Wg;
  ra.f32 = f32;
  ra.d_aux = grad->d_aux;
  ra.d_z = grad->d_z;
  ra.dlogits = dlogits;
  ra.dwmat = ec ? dlogits : nullptr;
  ra.dw_out = grad->dw;
  ra.dx = grad->dx;
  ++g_launches;
  if ((st = cuda_status(launch_router_bwd(ra, stream))) != MOE_OK) return st;

  GateWgradArgs wa{};
  wa.T = shape->T;
  wa.H = shape->H;
  wa.E = shape->E;
  wa.x = io->x;
  wa.f32 = f32;
  wa.dlogits = ra.dlogits;
  wa.dWg = grad->dWg;
  wa.dbg = grad->dbg;
  ++g_launches;
  return cuda_status(launch_gate_wgrad(wa, stream));
}

moe_status_t moe_forward_host(const moe_shape_t* shape, const moe_io_t* io, const void* x_host, float* out_host,
                              void* ws, size_t ws_bytes, cudaStream_t stream) {
  NvtxRange nvtx_range("moe_forward_host");
  moe_status_t st = check_shape(shape);
  if (st != MOE_OK) return st;
  if (io == nullptr || x_host == nullptr || out_host == nullptr || io->x == nullptr || io->out == nullptr)
    return MOE_ERR_INVALID_ARG;
  const size_t es = shape->dtype == MOE_DTYPE_BF16 ? 2 : 4;
  const size_t n = (size_t)shape->T * shape->H;
  if ((st = check_ws(shape, ws, ws_bytes)) != MOE_OK) return st;
  if (n > 0 && cudaMemcpyAsync(const_cast<void*>(io->x), x_host, n * es, cudaMemcpyHostToDevice, stream) != cudaSuccess)
    return MOE_ERR_CUDA;
  st = moe_forward(shape, io, ws, ws_bytes, stream);
  if (st != MOE_OK) return st;
  if (n > 0 && cudaMemcpyAsync(out_host, io->out, n * 4, cudaMemcpyDeviceToHost, stream) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

moe_status_t moe_get_device_status(void* ws, cudaStream_t stream) {
  if (ws == nullptr) return MOE_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return MOE_ERR_CUDA;
  int32_t word = 0;
  if (cudaMemcpy(&word, ws, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (word != 0) {
    const int32_t zero = 0;
    if (cudaMemcpy(ws, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return MOE_ERR_CUDA;
    return word == kDevBadIndex ? MOE_ERR_INVALID_ARG : MOE_ERR_TIMEOUT;
  }
  return MOE_OK;
}

void moe_set_wait_limit(long long cycles) { g_wait_limit = cycles > 0 ? cycles : 2000000000LL; }

void moe_set_kernel_options(int flags) {
  g_kernel_options.store(flags & (MOE_KERNEL_NO_CTA_PAIR | MOE_KERNEL_NO_TC_GATE | MOE_KERNEL_NO_TMA_ROUTER),
                         std::memory_order_relaxed);
}

int moe_get_kernel_options(void) { return g_kernel_options.load(std::memory_order_relaxed); }

moe_status_t moe_debug_activation(int activation, const float* u, float* out, int64_t n, cudaStream_t stream) {
  g_launches = 0;
  if (activation != MOE_ACT_GELU && activation != MOE_ACT_SILU) return MOE_ERR_INVALID_ARG;
  if (n < 0) return MOE_ERR_INVALID_ARG;
  if (n == 0) return MOE_OK;
  if (u == nullptr || out == nullptr) return MOE_ERR_INVALID_ARG;
  ++g_launches;
  return cuda_status(launch_activation_probe(activation, u, out, n, stream));
}

moe_status_t moe_debug_timeout_probe(void* ws, size_t ws_bytes, cudaStream_t stream) {
  g_launches = 0;
  if (ws == nullptr || ws_bytes < 256 || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MOE_ERR_INVALID_ARG;
  ++g_launches;
  return cuda_status(launch_timeout_probe(reinterpret_cast<int32_t*>(ws), g_wait_limit, stream));
}

int moe_last_launch_count(void) { return g_launches; }

const char* moe_status_string(moe_status_t s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape";
    case MOE_ERR_WORKSPACE: return "workspace too small";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

}  // extern "C"

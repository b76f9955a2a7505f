// Internal declarations shared by the kernels and the host C-ABI of the MoE forward library.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

constexpr int kChunk = 32;          // tokens per router chunk; also one warp in the permute ranks
constexpr int kRouterThreads = 256; // router block
constexpr int kRouterHC = 32;       // H columns per router pipeline stage
constexpr int kRouterStages = 4;

// Device error codes written to the workspace status word (first writer wins).
enum DevError : int {
  kDevOk = 0,
  kDevTimeoutProducer = 0x101,
  kDevTimeoutMma = 0x102,
  kDevTimeoutEpilogue = 0x103,
  kDevTimeoutProbe = 0x104,
  kDevTimeoutDrain = 0x105,
  kDevBadIndex = 0x201,  // an index array given by the caller held an out-of-range entry (it was skipped)
};

// Workspace sections (byte offsets from the workspace base, 256-aligned).
struct WsLayout {
  size_t status, offsets, cnt_pre, chunk_hist, chunk_base, loss_part, row_of, row_token, row_slot, x_perm, h, y,
      scores, tok_count, red_scratch, total;
  // training sections, after the inference ones: router logits [T,E] f32, pre-activation u, dout rows
  // (plain and weighted), du (all bf16), per-row dw partial sums, dlogits [T,E] f32
  size_t logits, u, dperm, dyperm, du, dwraw, dlogits, train_total;
  int nblk;       // router chunks = ceil(T / kChunk)
  long long rows; // rows of x_perm / h / y: T*k, or E*C under expert choice
  int ec_cap;     // C under expert choice, else 0
};

// Workspace word (next to the device error word) counting finished expert-choice selection blocks.
constexpr size_t kEcDoneOffset = 4;
// The same for the router (and histogram) blocks, whose last block runs the loss / dispatch reduction.
constexpr size_t kRouterDoneOffset = 8;
// ... and for the blocks of the multi-block reduction.
constexpr size_t kReduceDoneOffset = 12;

WsLayout ws_layout(const moe_shape_t& s);

struct ReduceArgs {
  int T, E, k, nblk;
  int ec_count;  // > 0: expert choice, every expert holds ec_count rows (no histogram, no dispatch)
  long long cap;  // < 0: unlimited
  const float* loss_part;
  int32_t* chunk_hist;  // [k][nblk][E]
  int32_t* chunk_base;  // [k][nblk][E] out: first rank of each chunk's assignments in its expert
  int32_t* cnt_pre;     // [E]
  int32_t* expert_counts;
  int32_t* offsets;     // [E+1]
  float* aux_loss;
  float* z_loss;
  int do_losses, do_dispatch;
  // scratch of the multi-block form (launch_reduce picks it for large k*nblk*E when these are given):
  // per-expert aux terms [E] (fp64), per-block z partials [256] and a finished-block counter (0
  // between calls)
  double* terms;
  float* zpart;
  unsigned* done;
};

struct RouterArgs {
  const void* x;
  const void* Wg;
  const void* bg;
  int T, H, E, k;
  int32_t* topk_idx;
  float* topk_w;
  float* loss_part;    // [nblk][E+1]: sum_t p[t,e] (E values) then sum_t lse_t^2
  int32_t* chunk_hist; // [k][nblk][E] or null
  // expert choice (non-null scores): no top-k; p goes to topk_w[T,E], logits to scores[E,T], and
  // tok_count[t] is cleared for the selection that follows
  float* scores;
  int32_t* tok_count;
  float* logits_out;  // training forward: logits [T,E] for the backward pass (else null)
  // [T,E] fp32 scratch: when given (bf16, E a multiple of 64) the gate is one tensor-core GEMM
  // into it, followed by the per-chunk softmax / top-k / partials kernel
  float* gemm_logits;
  int32_t* status;
  long long wait_limit;
  int num_sms;
  // When done is given, the last chunk block to finish also runs the loss / dispatch reduction of
  // red (in the router kernels that work chunk by chunk; launch_router reports whether it did).
  // done is a workspace counter that is 0 between calls.
  ReduceArgs red;
  unsigned* done;
};

struct EcSelectArgs {
  const float* scores;  // [E][T] router logits
  int T, E, C;
  int32_t* chosen;      // [E][C] out: chosen tokens, ascending
  int32_t* expert_counts;
  int32_t* cnt_pre;
  int32_t* tok_count;   // [T] experts that chose each token (cleared by the router)
  uint8_t* dropped;     // [T] out: 1 = chosen by no expert
  unsigned* done;       // finished-block counter, 0 between calls
};

struct EcGatherArgs {
  int32_t* status;  // device error word
  const void* x;
  int T, H, E, C, esize;
  const int32_t* chosen;  // [E][C]
  int32_t* offsets;       // [E+1] out: e*C
  int32_t* row_token;     // [E*C] out
  int32_t* row_slot;      // [E*C] out: the expert
  void* x_perm;           // [E*C][H] out
  float* out;             // [T][H] cleared; null: left alone (GEMM1 zeroes it)
};


struct ScatterArgs {
  int32_t* status;  // device error word
  const void* x;
  int T, H, E, k, nblk, esize;
  long long cap;
  const int32_t* topk_idx;
  const int32_t* chunk_base;
  const int32_t* offsets;
  uint8_t* dropped;
  int32_t* row_of;
  int32_t* row_token;
  int32_t* row_slot;
  void* x_perm;
  float* out;  // the chunk's rows cleared, split over its k slot blocks; null: left alone (GEMM1 clears it)
};

struct FfnArgs {
  int T, H, E, F, k;
  int rows_cap;  // height of x_perm / h / y: T*k, or E*C under expert choice
  long long avg_rows;  // expected rows per expert (T*k/E, or C), for the tile-shape choice
  const int32_t* offsets;
  const int32_t* row_token;
  const int32_t* row_slot;
  const float* topk_w;
  const void* x_perm;
  const void* W1;
  const void* b1;  // may be null (no bias)
  const void* W2;
  const void* b2;  // may be null (no bias)
  int act;         // moe_activation_t
  void* h;
  float* y;
  float* out;
  int fuse_combine;
  void* u_out;  // training forward: pre-activation u [rows, F] (bf16 path only; else null)
  int32_t* status;
  long long wait_limit;
  int num_sms;
  float* clear_out;  // [T, H] zeroed by GEMM1 (bf16, CTA-pair GEMM1 only: ffn_gemm1_on_pairs), or null
};

// ---- host-side helpers shared by the entry points (defined in moe_api.cu) ----
// Argument rules every entry point applies to a shape (the MOE_ERR_* codes of include/moe.h).
moe_status_t check_shape(const moe_shape_t* s);
// This host thread's count of kernels launched by the current moe_* call (moe_last_launch_count).
int& launch_count();
// Flags of moe_set_kernel_options (MOE_KERNEL_*), read at each launch.
int kernel_options();
// Bound on device-side waits (moe_set_wait_limit), read at each launch.
long long wait_limit();
// One NVTX range per entry-point call, named after the entry point.
struct NvtxRange {
  explicit NvtxRange(const char* name);
  ~NvtxRange();
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// Raises a kernel's dynamic shared-memory limit to at least `bytes` on the current device; the
// driver call is made once per (kernel, device) and size, so repeated launches cost nothing.
cudaError_t ensure_smem_limit(const void* kernel, int bytes);

// *reduced: whether the router's last block ran the reduction of a.red (a.done given), so that no
// separate reduce launch is needed
cudaError_t launch_router(const RouterArgs& a, int dtype, cudaStream_t st, int* launches, bool* reduced);
// Per-chunk histograms of a given topk_idx; with done given, the last block also runs the
// reduction of red when it fits one router-sized block (*reduced says whether it did; if not, a
// reduce launch must follow).
cudaError_t launch_hist(const int32_t* topk_idx, int T, int E, int k, int nblk, int32_t* chunk_hist, int32_t* status,
                        const ReduceArgs& red, unsigned* done, cudaStream_t st, bool* reduced);
cudaError_t launch_reduce(const ReduceArgs& a, cudaStream_t st);
cudaError_t launch_scatter(const ScatterArgs& a, int num_sms, cudaStream_t st);
cudaError_t launch_zero_outputs(int32_t* expert_counts, int E, float* aux, float* z, cudaStream_t st);
cudaError_t launch_loss_sums(const float* loss_part, const int32_t* cnt_pre, int nblk, int E, int T, float* sums,
                             cudaStream_t st);
cudaError_t launch_losses_from_sums(const float* sums, int E, float* aux, float* z, cudaStream_t st);
cudaError_t launch_ffn_f32(const FfnArgs& a, cudaStream_t st, int* launches);
cudaError_t launch_gate_logits_sm100(const void* x, const void* Wg, const void* bg, int T, int H, int E, float* logits,
                                     int32_t* status, long long wait_limit, int num_sms, cudaStream_t st);
cudaError_t launch_ec_select(const EcSelectArgs& a, cudaStream_t st);
// bf16, E in {64, 128, 256}, token choice: the gate GEMM with the softmax / top-k tail in its epilogue
cudaError_t launch_gate_router_sm100(const RouterArgs& a, cudaStream_t st);

// ---- backward pass ----
struct BwdPrepArgs {
  int T, H, E, F, k;
  int f32;            // storage dtype fp32: dperm / dyperm are written as fp32
  const int32_t* offsets;
  const int32_t* row_token;
  const int32_t* row_slot;
  const float* topk_w;
  const float* dout;  // [T,H]
  void* dperm;        // [rows,H] bf16 out
  void* dyperm;       // [rows,H] bf16 out
  float* dwraw;       // [rows] cleared
  float* dx;          // [T,H] cleared
  float* dWg;         // [H,E] cleared
  float* dbg;         // [E] cleared, or null
  float* db1;         // [E,F] cleared, or null
  float* db2;         // [E,H] cleared, or null
  float* dwmat;       // expert choice: [T,E] cleared, or null
};

struct BiasGradArgs {
  int H, F, E, k, rows_cap;
  int f32;         // du is fp32
  const int32_t* offsets;
  const int32_t* row_token;
  const int32_t* row_slot;
  const float* topk_w;
  const float* dout;
  const void* du;  // [rows,F] bf16
  float* db1;      // [E,F] or null
  float* db2;      // [E,H] or null
};

struct RouterBwdArgs {
  int T, H, E, k;
  const float* logits;  // [T,E] from the training forward
  const int32_t* topk_idx;
  const float* topk_w;
  const uint8_t* dropped;
  const int32_t* row_of;
  const int32_t* cnt_pre;
  const float* dwraw;
  const float* dout;
  const void* b2;  // [E,H] storage dtype, or null
  const void* Wg;  // [H,E] storage dtype
  int f32;         // storage dtype fp32
  float d_aux, d_z;
  float* dlogits;  // [T,E] out
  float* dw_out;   // [T,k] out (token choice) or [T,E] (expert choice), or null
  const float* dwmat;  // expert choice: [T,E] dL/dp of the chosen pairs (may alias dlogits), else null
  float* dx;       // [T,H] += Wg dlogits
};

struct GateWgradArgs {
  int T, H, E, chunk;
  int f32;  // x is fp32
  const void* x;
  const float* dlogits;
  float* dWg;
  float* dbg;  // or null
};

struct BwdGemmArgs {
  int T, H, E, F, k, rows_cap, act;
  long long avg_rows;
  const int32_t* offsets;
  const int32_t* row_token;
  const int32_t* row_slot;
  const float* topk_w;
  const void* W1;
  const void* W2;
  const void* x_perm;
  const void* h;
  const void* u;
  const void* dperm;
  const void* dyperm;
  void* du;
  float* dwraw;
  float* dx;
  float* dW1;
  float* dW2;
  int32_t* status;
  long long wait_limit;
  int num_sms;
};

struct EcDwArgs {
  int rows, H, E;
  const int32_t* row_token;
  const int32_t* row_slot;
  const float* dwraw;
  const float* dout;
  const void* b2;  // storage dtype, or null
  int f32;
  float* dwmat;    // [T,E]
};

cudaError_t launch_bwd_prep(const BwdPrepArgs& a, cudaStream_t st);
cudaError_t launch_ec_dw_scatter(const EcDwArgs& a, cudaStream_t st);
cudaError_t launch_bias_grad(const BiasGradArgs& a, cudaStream_t st);
cudaError_t launch_router_bwd(const RouterBwdArgs& a, cudaStream_t st);
cudaError_t launch_gate_wgrad(GateWgradArgs a, cudaStream_t st);
// dgrad of W2 (du, dw partials), dgrad of W1 (scatter-add into dx), weight gradients of W2 and W1
cudaError_t launch_bwd_gemms_sm100(const BwdGemmArgs& a, cudaStream_t st, int* launches);
// the same four GEMMs for fp32 storage, on CUDA cores
cudaError_t launch_bwd_gemms_f32(const BwdGemmArgs& a, cudaStream_t st, int* launches);
cudaError_t launch_ec_gather(const EcGatherArgs& a, cudaStream_t st);
cudaError_t launch_ec_combine(const float* y, const int32_t* chosen, const float* topk_w, int T, int E, int C, int H,
                              float* out, cudaStream_t st);
cudaError_t launch_ffn_bf16_sm100(const FfnArgs& a, cudaStream_t st, int* launches);
// Whether the bf16 FFN runs GEMM1 on CTA pairs (N = F, K = H, avg_rows rows per expert); its epilogue
// warps can then zero out during their first tile, in place of the scatter.
bool ffn_gemm1_on_pairs(int H, int F, long long avg_rows);
cudaError_t launch_combine(const float* y, const int32_t* row_of, const float* topk_w, int T, int H, int k, float* out,
                           cudaStream_t st);
cudaError_t launch_timeout_probe(int32_t* status, long long limit, cudaStream_t st);
// out[i] = act(u[i]), out[n + i] = act'(u[i]) with the tensor-core epilogues' arithmetic
cudaError_t launch_activation_probe(int act, const float* u, float* out, long long n, cudaStream_t st);

}  // namespace moe

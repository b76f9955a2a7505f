/*
 * moe.h -- C ABI of the B200 (sm_100a) sparse top-k Mixture-of-Experts layer: its forward pass,
 * its backward pass, and its losses over a batch split across data-parallel replicas.
 *
 * The layer (web page "MoE Training: Mixture of Experts", Quick Start "Basic MoE Architecture",
 * class MoELayer; Core Concepts 2-4; Advanced Patterns "Mixtral 8x7B Architecture") maps
 * x[T,H] to out[T,H] in four steps, each one entry point below:
 *
 *   moe_route       gate logits = x.Wg + bg, softmax, top-k, renormalised top-k weights,
 *                   Switch load-balancing loss and router z-loss           (Core Concepts 2, 3)
 *   moe_permute     per-expert counts, capacity, drop order, stable permutation of token rows
 *                   into expert-contiguous segments                        (Core Concepts 4;
 *                                                                           Best Practices 2)
 *   moe_expert_ffn  per-expert Linear(H,F) -> GELU -> Linear(F,H) as two grouped GEMMs
 *                   (Quick Start expert FFN), optionally with the weighted combine fused in;
 *                   SiLU and bias-free Linear layers for the Mixtral block's experts
 *   moe_combine     out[t] = sum over kept slots of w[t,s] * y[row(t,s)]     (Quick Start
 *                                                          "output[mask] += score * output";
 *                                                          Mixtral block index_add_)
 *   moe_forward     the four chained on one stream (fused combine)
 *
 * Around them: moe_forward_host (the same pass on host buffers, copies included), moe_route_noalloc
 * (the router without a workspace), moe_forward_train + moe_backward (every gradient of the layer),
 * moe_loss_sums + moe_losses_from_sums (the losses of a batch spread over replicas).
 *
 * Two routing rules (moe_shape_t.routing): token choice, where every token takes its top-k experts
 * (Quick Start; Core Concepts 2 top-1 / top-2), and expert choice, where every expert takes its
 * top-C tokens (Core Concepts 2, "Expert Choice Routing").  The buffers whose meaning differs
 * between the two are listed under moe_io_t.
 *
 * Conventions shared by every entry point
 *  - All tensors are row-major and contiguous.  Every pointer in moe_io_t is a DEVICE pointer
 *    owned by the caller; the library never allocates device memory and never frees it.
 *  - Storage dtype (moe_shape_t.dtype) applies to x, Wg, bg, W1, b1, W2, b2: MOE_DTYPE_F32 or
 *    MOE_DTYPE_BF16.  Accumulation is fp32 everywhere.  out, topk_w and the losses are fp32.
 *  - The biases bg, b1 and b2 are optional: a NULL pointer means the Linear layer has no bias
 *    (the Mixtral block's gate and experts are Linear(..., bias=False)), computed as a zero bias.
 *  - All work is asynchronous on the given stream (0 = legacy default stream).  No entry point
 *    synchronises except moe_get_device_status.
 *  - Arguments are validated on the host before anything is launched:
 *      MOE_ERR_INVALID_ARG  null shape/io/workspace pointer, a needed io pointer that is null, a
 *                           device pointer of x/Wg/W1/W2/out/workspace not 16-byte aligned,
 *                           T < 0, H/E/F/k <= 0, k > E, k > 8, E > 256, capacity_factor <= 0 or
 *                           NaN, min_capacity < 0, unknown dtype, activation or routing, a non-null b1/b2 not 16-byte
 *                           aligned
 *      MOE_ERR_UNSUPPORTED  bf16 with H or F not a multiple of 64; f32 with H or F not a multiple
 *                           of 4; rows*max(H,F) beyond 2^31 elements (rows = T*k, or E*C under
 *                           expert choice)
 *      MOE_ERR_WORKSPACE    ws_bytes < moe_workspace_size(shape)
 *      MOE_ERR_CUDA         a launch or driver call failed (the CUDA error is not cleared)
 *    On any error nothing has been launched by that call.
 *  - The workspace is a caller-allocated device buffer of moe_workspace_size() bytes, 256-byte
 *    aligned, whose first 256 bytes (the device error word) must be zero before its first use
 *    (e.g. cudaMemsetAsync(ws, 0, 256, stream)); afterwards the library keeps them.  It carries state from moe_route to moe_permute to moe_expert_ffn to moe_combine, so
 *    one workspace serves one layer invocation at a time; calls on distinct workspaces are
 *    independent and may run concurrently on different streams.
 *  - T = 0 is valid: every entry point returns MOE_OK; moe_route writes aux_loss = z_loss = 0 and
 *    moe_permute writes expert_counts = 0.
 *  - Device-side waits (pipeline barriers in the tensor-core kernels) are bounded.  A wait that
 *    runs out records an error word in the workspace and the kernel returns early;
 *    moe_get_device_status() reports it as MOE_ERR_TIMEOUT.  No kernel traps.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,
  MOE_ERR_UNSUPPORTED = 2,
  MOE_ERR_WORKSPACE = 3,
  MOE_ERR_CUDA = 4,
  MOE_ERR_TIMEOUT = 5
} moe_status_t;

typedef enum { MOE_DTYPE_F32 = 0, MOE_DTYPE_BF16 = 1 } moe_dtype_t;

/* Routing rule.  Expert choice: the router's logits are read per expert (the page transposes
 * them to (experts, tokens)) and every expert takes the C tokens with the largest logits, ties to
 * the lower token index, C = min(T, max(ceil(capacity_factor * T * k / E), min_capacity)) -- k is then the average
 * number of experts per token, and capacity_factor = +INFINITY gives C = T.  Each chosen
 * (token, expert) pair is weighted by the token's softmax probability over the experts, not
 * renormalised; a token chosen by no expert gets out = 0.  Every expert holds exactly C rows. */
typedef enum { MOE_ROUTING_TOKEN_CHOICE = 0, MOE_ROUTING_EXPERT_CHOICE = 1 } moe_routing_t;

/* Activation between the two expert Linear layers.  GELU is the exact erf form (Quick Start
 * expert, nn.GELU()); SiLU is u * sigmoid(u) (Advanced Patterns, Mixtral block experts). */
typedef enum { MOE_ACT_GELU = 0, MOE_ACT_SILU = 1 } moe_activation_t;

/* Problem statement.  capacity_factor = +INFINITY means dropless.  Per-expert capacity is
 * max(ceil(capacity_factor * T * k / E), min_capacity) evaluated in double ("MoE Training" page,
 * Core Concepts 4 and Best Practices 2 give capacity = tokens * CF / E; k counts the assignments of
 * top-k routing). */
typedef struct {
  int32_t T;              /* tokens (batch * sequence), >= 0 */
  int32_t H;              /* hidden size */
  int32_t E;              /* experts, 1..256 */
  int32_t F;              /* FFN width of each expert */
  int32_t k;              /* experts per token, 1..min(E, 8) */
  double capacity_factor; /* > 0; +INFINITY = no capacity limit */
  moe_dtype_t dtype;      /* storage type of x and all weights */
  moe_activation_t activation; /* expert activation; a zero-initialised shape gets GELU */
  moe_routing_t routing;       /* a zero-initialised shape gets token choice */
  int32_t min_capacity;        /* lower bound on the per-expert capacity ("min_capacity" of the page's
                                  Core Concepts 4 configuration); 0 = none, < 0 invalid */
} moe_shape_t;

/* Caller-owned device buffers.  Layouts (row-major):
 *   x[T,H] Wg[H,E] bg[E] W1[E,H,F] b1[E,F] W2[E,F,H] b2[E,H]       storage dtype, read only;
 *                                                                  bg, b1, b2 may be NULL
 *   out[T,H]           fp32  layer output
 *   topk_idx[T,k]      int32 chosen experts, slot s = rank s by (logit desc, expert index asc)
 *   topk_w[T,k]        fp32  softmax probabilities of the chosen experts divided by their sum
 *                            (pre-drop values; dropped slots keep their weight here)
 *   expert_counts[E]   int32 kept assignments per expert (after capacity)
 *   dropped[T,k]       uint8 1 = assignment dropped by capacity
 *   aux_loss, z_loss   fp32 scalars: E*sum_e f_e*P_e and mean_t logsumexp_t^2, no coefficients
 * Under expert choice (C as above) four of them change shape and meaning:
 *   topk_idx[E,C]      int32 the tokens each expert chose, in ascending token order
 *   topk_w[T,E]        fp32  softmax probabilities of every token over all experts (the weight of
 *                            (t,e) when e chose t)
 *   expert_counts[E]   int32 C for every expert
 *   dropped[T]         uint8 1 = token chosen by no expert
 * and aux_loss = sum_e P_e (f_e = 1/E; 1 up to rounding). */
typedef struct {
  const void* x;
  const void* Wg;
  const void* bg;
  const void* W1;
  const void* b1;
  const void* W2;
  const void* b2;
  float* out;
  int32_t* topk_idx;
  float* topk_w;
  int32_t* expert_counts;
  uint8_t* dropped;
  float* aux_loss;
  float* z_loss;
} moe_io_t;

/* Pointers into a workspace, for inspection of the intermediate stages. */
typedef struct {
  int32_t* status;     /* device error word (0 = ok) */
  int32_t* offsets;    /* [E+1] exclusive prefix sum of expert_counts; offsets[E] = kept rows */
  int32_t* cnt_pre;    /* [E] assignments per expert before capacity */
  int32_t* row_of;     /* [T,k] row of assignment (t,s) in x_perm, -1 if dropped */
  int32_t* row_token;  /* [T*k] token of each row (rows >= offsets[E] unused) */
  int32_t* row_slot;   /* [T*k] slot of each row */
  void* x_perm;        /* [T*k, H] storage dtype: x rows grouped by expert, (slot, token) order */
  void* h;             /* [T*k, F] storage dtype: act(x_perm . W1[e] + b1[e]) */
  float* y;            /* [T*k, H] fp32: h . W2[e] + b2[e] (only written when the combine is not fused) */
  size_t bytes;        /* total workspace size */
  float* scores;       /* expert choice only (else NULL): [E,T] fp32 router logits, expert-major */
} moe_ws_view_t;
/* Under expert choice the row buffers hold E*C rows instead of T*k, row e*C + j being the j-th token
 * that expert e chose; row_slot holds the expert and row_of is unused. */

/* Workspace bytes for a shape; 0 if the shape is invalid.  Host only, pure. */
MOE_API size_t moe_workspace_size(const moe_shape_t* shape);

/* Per-expert capacity the shape implies.  Token choice: max(ceil(capacity_factor * T * k / E),
 * min_capacity), or -1 when capacity_factor = +INFINITY (no limit).  Expert choice: C = min(T,
 * max(ceil(capacity_factor * T * k / E), min_capacity)), the number of tokens every expert takes
 * (the leading size of topk_idx[E,C]).
 * -2 if the shape is invalid.  Host only, pure. */
MOE_API int64_t moe_capacity(const moe_shape_t* shape);

/* Pointers to each stage buffer inside `ws` for `shape`.  Host only, pure. */
MOE_API moe_status_t moe_workspace_layout(const moe_shape_t* shape, void* ws, moe_ws_view_t* view);

/* Router ("MoE Training" page, Quick Start MoELayer.forward: gate, softmax, topk, renormalise;
 * Core Concepts 3: load_balancing_loss, router_z_loss).
 * Reads x, Wg, bg.  Writes topk_idx, topk_w, aux_loss, z_loss (and router partials in ws).
 * Token choice: 1 launch, the gate with its softmax / top-k tail, whose last block to finish also
 * reduces the loss partials (a workspace counter beside the error word picks that block) when they
 * are small enough, k*ceil(T/32)*E <= 4096; else one reduce launch follows.  bf16
 * layers with 8 or 16 experts stream x through a shared-memory ring of bulk copies into mma.sync
 * (32 experts: register-fed mma.sync); bf16 layers whose expert count is a multiple of 64 run the
 * gate as a tcgen05 GEMM into the workspace followed by the per-chunk softmax / top-k (one launch
 * more), or -- with 64, 128 or 256 experts and at least one 128-token tile per two SMs -- as one
 * tcgen05 GEMM whose epilogue does the softmax / top-k, followed by one reduce launch.
 * Expert choice: also the per-expert selection (Core Concepts 2), so it writes the chosen tokens
 * to topk_idx[E,C], expert_counts and dropped[T] as well; 3 launches, one more for bf16 layers whose
 * expert count is a multiple of 64. */
MOE_API moe_status_t moe_route(const moe_shape_t* shape, const moe_io_t* io, void* ws, size_t ws_bytes,
                       cudaStream_t stream);

/* moe_route without a workspace, for callers that cannot allocate device memory: code running
 * inside another runtime's fixed device-memory pool, serving paths that forbid any device
 * allocation after start-up, plugins whose host framework owns every allocation.  The pages
 * have no counterpart; it exists for these callers only.
 * Same inputs, outputs, validation and results as moe_route.  The router's scratch (per-block
 * sums, per-chunk histograms, and a device error word where a bounded wait of the tensor-core gate
 * would record a timeout, which this call has no way to report) lives in a 1 MiB array built into
 * the library, which every GPU that loads the library keeps until the process exits.  It needs
 *   256 + align256(ceil(T/32)*(E+1)*4) + align256(k*ceil(T/32)*E*4) + align256(E*4) <= 1 MiB
 * (for example T = 16384 with E = 64, k = 2 uses 395 KB); larger shapes return MOE_ERR_WORKSPACE
 * before anything is launched.  No device memory is allocated or freed, by this call or by any
 * routine it calls.  The first call on a device looks up the array's device address for that
 * device (cudaGetSymbolAddress, with the device current); make that first call before any stream
 * capture.  Later calls made outside stream capture look the address up again, so a context that
 * was reset and rebuilt (cudaDeviceReset) is served its new address.  Every call, on every stream,
 * shares the one array and leaves the last call's contents in it: calls that overlap on the GPU
 * race, so serialise them (one stream, or events).  1 launch (2 with the one-GEMM gate of 64, 128
 * or 256 experts, or when k*ceil(T/32)*E > 4096: the reduction is then a launch of its own); one
 * NVTX range.
 * Token choice only: an expert-choice shape returns MOE_ERR_UNSUPPORTED. */
MOE_API moe_status_t moe_route_noalloc(const moe_shape_t* shape, const moe_io_t* io, cudaStream_t stream);

/* Losses of a batch split over data-parallel replicas ("MoE Training" page, Core Concepts 3:
 * load_balancing_loss, router_z_loss).  Both losses are built from sums over tokens:
 *   aux = E * sum_e (cnt_e / sum_e' cnt_e') * (Psum_e / T),   z = Zsum / T,
 * with cnt_e the assignments routed to expert e before any drop (T*k in all under token choice,
 * E*C under expert choice), Psum_e = sum_t p[t,e] and Zsum = sum_t lse_t^2.  Each sum is additive
 * over disjoint token sets, so adding the replicas' sums (an all-reduce) and applying the formula
 * gives the losses of the whole batch -- which a mean of the replicas' own aux values does not,
 * as aux is a product of two means.
 *
 * moe_loss_sums: after moe_route, moe_forward or moe_forward_train on ws (same shape, same stream),
 * writes the 2E+2 fp32 sums of this call's batch to the device buffer sums (caller-owned, 4-byte
 * aligned): sums[0..E) = cnt_e, sums[E..2E) = Psum_e, sums[2E] = Zsum, sums[2E+1] = T.  Counts and
 * T are exact below 2^24.  T = 0 gives zeros.  Errors: MOE_ERR_INVALID_ARG (null sums or bad
 * shape), MOE_ERR_WORKSPACE, MOE_ERR_CUDA.  One launch.
 *
 * moe_losses_from_sums: aux_loss and z_loss (device fp32 scalars) from 2E+2 sums laid out as above
 * -- one replica's, or their element-wise total over replicas.  A total of T = 0 gives zeros.
 * Errors: MOE_ERR_INVALID_ARG (E outside [1, 256] or a null pointer), MOE_ERR_CUDA.  One launch. */
MOE_API moe_status_t moe_loss_sums(const moe_shape_t* shape, void* ws, size_t ws_bytes, float* sums,
                           cudaStream_t stream);
MOE_API moe_status_t moe_losses_from_sums(int E, const float* sums, float* aux_loss, float* z_loss,
                                  cudaStream_t stream);

/* Dispatch (Core Concepts 4 "capacity_factor", "drop_tokens"; Best Practices 2; Advanced Patterns
 * Mixtral block gather by expert).  Assignments are visited slot-major then by token; an
 * assignment is kept iff fewer than `capacity` earlier assignments went to its expert.
 * Reads x, topk_idx.  Writes expert_counts, dropped, the row maps and x_perm in ws, and clears
 * out[T,H] to zero (the fused combine accumulates into it).  Token choice: 2 launches, per-chunk
 * histograms (the last block also scans them into offsets, when k*ceil(T/32)*E <= 4096; else a
 * reduce launch follows) and the scatter; expert choice: 1.  The kernels check every index they
 * read from topk_idx (see moe_get_device_status); nothing outside the buffers is touched.
 * Expert choice: nothing is dropped (each expert already holds exactly C tokens); reads x and
 * topk_idx[E,C], writes the row maps and x_perm, and clears out. */
MOE_API moe_status_t moe_permute(const moe_shape_t* shape, const moe_io_t* io, void* ws, size_t ws_bytes,
                         cudaStream_t stream);

/* Expert FFN (Quick Start expert: Linear(H, F) -> GELU(erf) -> Linear(F, H), with biases) as two
 * grouped GEMMs over the expert segments of x_perm.  bf16: tcgen05 tensor cores, h stored bf16;
 * f32: CUDA cores, h stored f32.  fuse_combine != 0: out[t] += topk_w[t,s]*(h.W2[e] + b2[e]) for
 * every kept row (out must hold zeros from moe_permute); at most k fp32 adds reach each element,
 * so for k <= 2 the result does not depend on their order (under expert choice up to E adds
 * reach an element, in no fixed order).  fuse_combine == 0: y in ws is
 * written instead and out is untouched.  Reads W1, b1, W2, b2, topk_w and the ws state of
 * moe_permute. */
MOE_API moe_status_t moe_expert_ffn(const moe_shape_t* shape, const moe_io_t* io, void* ws, size_t ws_bytes,
                            int fuse_combine, cudaStream_t stream);

/* Combine from a materialised y (Quick Start "output[mask] += expert_scores * expert_output"):
 * out[t] = sum over kept slots s, in slot order, of topk_w[t,s] * y[row_of(t,s)]; tokens with
 * every slot dropped get zeros.  Overwrites out.  Use after moe_expert_ffn(fuse_combine = 0).
 * Expert choice: out[t] = sum over the experts that chose t, in ascending expert order, of
 * topk_w[t,e] * y[row(t,e)], the row found in the expert's ascending topk_idx[e,:]; a token that no
 * expert chose gets zeros.  Overwrites out, with no atomics: both rules give the same bits on every
 * run.  Reads topk_idx as well. */
MOE_API moe_status_t moe_combine(const moe_shape_t* shape, const moe_io_t* io, void* ws, size_t ws_bytes,
                         cudaStream_t stream);

/* moe_route, moe_permute and moe_expert_ffn(fuse_combine = 1) on one stream.  Where bf16 GEMM1 runs
 * on CTA pairs (F a multiple of 256, H of 128, T*k/E >= 256 or under expert choice C >= 256, pairs
 * not switched off with moe_set_kernel_options), its epilogue warps zero out during their first
 * tile and the scatter (or gather) leaves out alone; the result is the same.  Token choice: the gate
 * (whose last block reduces the losses and the dispatch), the scatter, GEMM1 and GEMM2: 4 launches,
 * one more for either tensor-core gate form of moe_route or when the reduction does not fit the
 * gate's last block (k*ceil(T/32)*E > 4096).  Expert choice: 6 launches, 7 with the
 * two-kernel tensor-core gate. */
MOE_API moe_status_t moe_forward(const moe_shape_t* shape, const moe_io_t* io, void* ws, size_t ws_bytes,
                         cudaStream_t stream);

/* The same forward pass for callers whose activations live in host memory: copies x_host
 * (T*H elements of the storage dtype) to io->x, runs moe_forward, and copies io->out back to
 * out_host (T*H fp32), all asynchronously on `stream` (pinned host memory makes the copies
 * asynchronous).  io->x must be a writable device buffer.  Does not synchronise. */
MOE_API moe_status_t moe_forward_host(const moe_shape_t* shape, const moe_io_t* io, const void* x_host,
                              float* out_host, void* ws, size_t ws_bytes, cudaStream_t stream);

/* ---------------------------------------------------------------------------------------------
 * Training: forward pass that keeps what the backward pass needs, and the backward pass.
 * The pages train MoE layers (Core Concepts 3 adds the two losses to the training loss); the
 * gradients are the chain rule through the forward definition: for L with dL/dout = dout,
 * dL/daux = d_aux and dL/dz = d_z, every input x, Wg, bg, W1, b1, W2, b2 gets dL/d(input).  The
 * top-k choice and the capacity drops are piecewise constant and carry no gradient; a dropped
 * slot contributes nothing.  Both storage types (bf16: tensor cores, intermediates in bf16; fp32:
 * CUDA cores, intermediates in fp32) and both routing rules.  Under
 * expert choice the weight of a chosen pair is the softmax probability itself, so the gate receives
 * p (dw - sum p dw) with no renormalisation term, and the aux-loss term cancels (f_e = 1/E).
 * ------------------------------------------------------------------------------------------- */

/* Caller-owned device buffers of the backward pass, fp32, row-major. */
typedef struct {
  const float* dout; /* [T,H] dL/dout */
  float d_aux;       /* dL/d aux_loss (its coefficient in the loss) */
  float d_z;         /* dL/d z_loss */
  float* dx;         /* [T,H] */
  float* dWg;        /* [H,E] */
  float* dbg;        /* [E]; must be NULL exactly when io->bg is NULL */
  float* dW1;        /* [E,H,F] */
  float* db1;        /* [E,F]; NULL exactly when io->b1 is NULL */
  float* dW2;        /* [E,F,H] */
  float* db2;        /* [E,H]; NULL exactly when io->b2 is NULL */
  float* dw;         /* optional (may be NULL): dL/d topk_w -- [T,k] per slot, 0 for dropped slots;
                        under expert choice [T,E], 0 for pairs not chosen */
} moe_grad_t;

/* Workspace bytes for moe_forward_train + moe_backward (the inference layout plus the saved router
 * logits, the pre-activation u and the backward's row buffers); 0 if the shape is invalid.  A
 * training workspace also serves every inference entry point. */
MOE_API size_t moe_train_workspace_size(const moe_shape_t* shape);

/* moe_forward (same outputs), also keeping the router logits and the pre-activation u in ws for
 * moe_backward.  ws_bytes >= moe_train_workspace_size(shape).  Launches as moe_forward. */
MOE_API moe_status_t moe_forward_train(const moe_shape_t* shape, const moe_io_t* io, void* ws, size_t ws_bytes,
                               cudaStream_t stream);

/* Gradients of the layer after moe_forward_train on the same ws, io and inputs.  Reads x, Wg, W1,
 * W2, b2 (optional), topk_idx, topk_w, dropped from io and the saved state from ws; writes every
 * buffer of grad (dx, dWg, dbg are cleared first; no output is accumulated across calls).
 * Row order of the bf16 intermediates: the permuted (expert-major) rows of the forward pass.
 * Order of fp32 additions in dx, dWg and dbg is not fixed (atomics).  7 or 8 launches (one more
 * under expert choice). */
MOE_API moe_status_t moe_backward(const moe_shape_t* shape, const moe_io_t* io, const moe_grad_t* grad, void* ws,
                          size_t ws_bytes, cudaStream_t stream);

/* Synchronises `stream`, then reads and clears the workspace's device error word.
 * Returns MOE_OK, MOE_ERR_TIMEOUT (a bounded device wait ran out), MOE_ERR_INVALID_ARG (a kernel met
 * an out-of-range entry in a caller-supplied index array -- an expert outside [0, E) in topk_idx, or
 * a token outside [0, T) in an expert-choice topk_idx -- and skipped it: such a slot counts as dropped,
 * such a row computes on zeros for token 0; results are then not meaningful) or MOE_ERR_CUDA. */
MOE_API moe_status_t moe_get_device_status(void* ws, cudaStream_t stream);

/* Bound on device-side waits, in GPU clock cycles (default 2e9, about one second).  Applies to
 * launches made after the call.  Values <= 0 restore the default. */
MOE_API void moe_set_wait_limit(long long cycles);

/* ---- expert parallelism ("MoE Training" page, Core Concepts 4, "Expert Parallelism": the experts
 * are spread over workers, every kept assignment's row travels to the worker that holds its expert,
 * and the expert outputs travel back to be combined where the token lives).  Each worker routes and
 * permutes its own tokens with moe_route / moe_permute over all E experts; the rows of expert e then
 * form the contiguous segment [offsets[e], offsets[e+1]) of its x_perm (moe_workspace_layout).  The
 * two calls below move those segments and run the owner's experts on what it received; the worker
 * that sent them writes the returned rows into its y and finishes with moe_combine.  A segment
 * table is the whole exchange plan, so the same calls serve any placement of experts on workers. */

/* One contiguous run of rows to copy: `rows` rows of the call's row_bytes each, from src to dst.
 * src and dst are device pointers, 16-byte aligned; either may be another GPU's memory mapped into
 * this one (a peer-accessible allocation), which makes the copy a pull or a push over NVLink. */
typedef struct {
  const void* src;
  void* dst;
  int64_t rows;
} moe_row_segment_t;

/* Copies every segment of segs[nsegs] (a DEVICE array of moe_row_segment_t, 16-byte aligned) in one
 * launch: the dispatch of every row a worker receives, or the return of every row it sends back.
 * row_bytes: bytes per row, a positive multiple of 16 (H * 2 for bf16 x rows, H * 4 for fp32 y rows).
 * max_rows: an upper bound on any segment's rows (it sizes the grid; longer segments are still copied
 * whole).  Segments must not overlap each other's destinations.  A segment whose src or dst is not
 * 16-byte aligned is skipped and, when status is not NULL, recorded there as MOE_ERR_INVALID_ARG's
 * device code (status: a device int32, e.g. a workspace's error word).  Returns MOE_ERR_INVALID_ARG
 * for nsegs < 0 or > 65535, a bad row_bytes or max_rows, or a NULL / misaligned table with nsegs > 0;
 * nothing is launched for nsegs = 0.  1 launch. */
MOE_API moe_status_t moe_copy_row_segments(const moe_row_segment_t* segs, int nsegs, int64_t row_bytes,
                                           int64_t max_rows, int32_t* status, cudaStream_t stream);

/* The grouped expert FFN over caller-given rows (Quick Start expert Linear(H,F) -> act -> Linear(F,H),
 * every expert on its own segment): for each expert e < shape->E and each row r in
 * [offsets[e], offsets[e+1]),
 *     y[r,:] = act(x_rows[r,:] . W1[e] + b1[e]) . W2[e] + b2[e]      (fp32, not weighted)
 * shape: H, F, E (the experts held in W1[E,H,F], b1[E,F], W2[E,F,H], b2[E,H], e.g. one worker's
 * share of the layer's experts), dtype and activation are used; T, k, capacity and routing are not.
 * x_rows[rows_cap,H] (storage dtype) and y[rows_cap,H] are device buffers; offsets[E+1] is a device
 * int32 array, non-decreasing from 0, offsets[E] <= rows_cap.  Offsets that break this are clamped
 * on the device (and recorded in the workspace's error word, reported by moe_get_device_status),
 * so no row outside [0, rows_cap) is read or written.  Rows in [offsets[E], rows_cap) of y are not
 * written.  Workspace: moe_expert_ffn_rows_workspace_size(shape, rows_cap) bytes, 256-byte aligned,
 * first 256 bytes zero before its first use; it holds the bf16 / fp32 h rows.  Validation as for
 * moe_expert_ffn (H, F, E, dtype, activation; rows_cap >= 0; rows_cap * max(H, F) < 2^31).
 * 3 launches (offsets check, GEMM1, GEMM2). */
MOE_API size_t moe_expert_ffn_rows_workspace_size(const moe_shape_t* shape, int64_t rows_cap);
MOE_API moe_status_t moe_expert_ffn_rows(const moe_shape_t* shape, int64_t rows_cap, const int32_t* offsets,
                                         const void* x_rows, const void* W1, const void* b1, const void* W2,
                                         const void* b2, float* y, void* ws, size_t ws_bytes, cudaStream_t stream);

/* Kernel-selection switches for side-by-side comparisons of the kernels; normal use needs none.
 *   MOE_KERNEL_NO_CTA_PAIR  single-CTA 128-row grouped-GEMM tiles everywhere, instead of the CTA-pair
 *                           256 x 256 tiles the long-segment shapes use (forward and backward GEMMs)
 *   MOE_KERNEL_NO_TC_GATE   the CUDA-core gate kernels instead of the tensor-core ones (mma.sync for
 *                           8/16/32 experts, the tcgen05 GEMM for multiples of 64)
 *   MOE_KERNEL_NO_TMA_ROUTER  for bf16 with 8 or 16 experts, the register-direct mma.sync gate (x loaded
 *                           into registers) instead of the one that streams x through a shared-memory
 *                           ring of bulk copies
 * Default 0.  Process-wide; applies to launches made after the call, from any host thread.  Results
 * stay within the same tolerances of the definition either way; unknown bits are ignored. */
typedef enum {
  MOE_KERNEL_DEFAULT = 0,
  MOE_KERNEL_NO_CTA_PAIR = 1,
  MOE_KERNEL_NO_TC_GATE = 2,
  MOE_KERNEL_NO_TMA_ROUTER = 4
} moe_kernel_flags_t;
MOE_API void moe_set_kernel_options(int flags);
MOE_API int moe_get_kernel_options(void);

/* The bf16 tensor-core epilogues' activation arithmetic on n given fp32 values: out[i] = act(u[i])
 * and out[n + i] = act'(u[i]), with act the shape's GELU (u Phi(u), Phi from Abramowitz & Stegun
 * 7.1.26) or SiLU.  For tests of that arithmetic against its definition.  u: n floats, out: 2n
 * floats, both device memory.  Errors: MOE_ERR_INVALID_ARG (unknown activation, n < 0, a null
 * pointer with n > 0), MOE_ERR_CUDA.  One launch (none for n = 0). */
MOE_API moe_status_t moe_debug_activation(int activation, const float* u, float* out, int64_t n, cudaStream_t stream);

/* Launches one block that waits on a pipeline barrier nothing will ever complete, with the
 * current wait bound; it must come back with the error word set.  For testing the timeout path. */
MOE_API moe_status_t moe_debug_timeout_probe(void* ws, size_t ws_bytes, cudaStream_t stream);

/* Number of kernels the last moe_* call launched on the host thread (for launch accounting). */
MOE_API int moe_last_launch_count(void);

MOE_API const char* moe_status_string(moe_status_t status);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */

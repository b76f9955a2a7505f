// Router, loss/dispatch reduction and permutation kernels of the MoE forward pass.
//
// Router ("MoE Training: Mixture of Experts" page, Quick Start MoELayer.forward; Core Concepts 2
// "Routing Mechanisms" and 3 "Load Balancing"):
//   logits = x.Wg + bg (bg optional), p = softmax(logits), top-k by (logit desc, index asc), w = p_sel / sum p_sel,
//   aux = E * sum_e f_e P_e (f from pre-drop counts / (T*k), P = mean_t p), z = mean_t lse_t^2.
// Dispatch (Core Concepts 4 capacity_factor / drop_tokens; Best Practices 2 capacity tuning):
//   capacity = ceil(CF*T*k/E) or unlimited; assignments ranked per expert in (slot, token) order;
//   rank < capacity kept; the rank is also the row inside the expert's segment.
#include <cuda_bf16.h>
#include <float.h>
#include <math.h>
#include <stdlib.h>

#include "moe_internal.cuh"
#include "sm100_ptx.cuh"

namespace moe {

namespace {

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, int src_bytes) {
  uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// Shared-memory plan of the router block (bytes).
struct RouterSmem {
  int xrow;     // bytes per staged x row (HC elements + 16 pad)
  int xstage;   // bytes of one x stage (32 rows)
  int wstage;   // bytes of one Wg stage (HC x E elements, 16-aligned)
  int epad;     // E rounded up to 4
  int logits;   // offset of logits[32][epad] floats
  int red;      // offset of K-split partials
  int psum;     // offset of per-warp softmax sums [8][epad]
  int misc;     // offset of small scratch (hist, z)
  int total;
};

__host__ __device__ inline RouterSmem router_smem(int E, int esize) {
  RouterSmem s;
  s.epad = (E + 3) & ~3;
  s.xrow = kRouterHC * esize + 16;
  s.xstage = kChunk * s.xrow;
  s.wstage = ((kRouterHC * E * esize) + 15) & ~15;
  int stages = kRouterStages * (s.xstage + s.wstage);
  s.logits = (stages + 15) & ~15;
  s.red = s.logits + kChunk * s.epad * 4;
  int pairs = 8 * (s.epad / 4);
  int ks = pairs >= kRouterThreads ? 1 : kRouterThreads / pairs;
  int red_bytes = ks > 1 ? ks * kChunk * s.epad * 4 : 0;
  s.psum = s.red + red_bytes;
  s.misc = s.psum + 8 * s.epad * 4;
  s.total = s.misc + (8 * 256 + 64) * 4;  // hist[k<=8][E<=256] ints + z per warp
  return s;
}

constexpr int kRB = 16;  // loads per batch in the reduction below

// Shared memory of the reduction below, for a block of NT threads.
template <int NT>
struct ReduceSmem {
  int gsum[NT];
  int cnt_s[256];
  double term[256];
  float zred[32];
  float pf[NT];
  float zf[NT];
};

// One block of NT threads (E <= NT): losses from the router partials, per-expert totals, capacity,
// offsets and the exclusive scan of the chunk histograms in (slot, chunk) order.  The partials are
// read through L2 (__ldcg): in the fused form other blocks of the same grid wrote them.  Every sum
// runs in a fixed order, so a given NT gives the same bits on every run.
template <int NT>
__device__ void reduce_body(const ReduceArgs& a, ReduceSmem<NT>& sm) {
  int* gsum = sm.gsum;
  int* cnt_s = sm.cnt_s;
  double* term = sm.term;
  float* zred = sm.zred;
  float* pf = sm.pf;
  float* zf = sm.zf;
  const int tid = threadIdx.x, E = a.E;
  const int C = a.k * a.nblk;  // chunks in (slot, token-chunk) order
  const int G = NT / E;        // groups of chunks
  const int g = tid / E, e = tid % E;
  const bool in = tid < G * E;
  const bool tc = a.ec_count <= 0;
  const int c0 = in ? (int)((long long)C * g / G) : 0;
  const int c1 = in ? (int)((long long)C * (g + 1) / G) : 0;
  const int b0 = in ? (int)((long long)a.nblk * g / G) : 0;
  const int b1 = in ? (int)((long long)a.nblk * (g + 1) / G) : 0;

  // The first kRB values of every range this thread reads, all loads issued together (with short
  // ranges that is every load: one L2 round trip); longer ranges continue in batches of kRB
  // independent loads.  The additions keep their order (index ascending).
  int hv[kRB];
  float pv[kRB], zv[kRB];
#pragma unroll
  for (int u = 0; u < kRB; ++u) {
    hv[u] = tc && c0 + u < c1 ? __ldcg(&a.chunk_hist[(size_t)(c0 + u) * E + e]) : 0;
    pv[u] = a.do_losses && b0 + u < b1 ? __ldcg(&a.loss_part[(size_t)(b0 + u) * (E + 1) + e]) : 0.f;
    zv[u] = a.do_losses && tid + u * NT < a.nblk ? __ldcg(&a.loss_part[(size_t)(tid + u * NT) * (E + 1) + E]) : 0.f;
  }
  if (a.do_losses) {
    // P_e: thread (g, e) sums a fixed range of router blocks, then the group sums are added in
    // group order; z: thread-strided sums then a fixed tree.  Same order on every run.
    float ps = 0.f;
#pragma unroll
    for (int u = 0; u < kRB; ++u)
      if (b0 + u < b1) ps += pv[u];
    for (int b = b0 + kRB; b < b1; b += kRB) {
      float v[kRB];
#pragma unroll
      for (int u = 0; u < kRB; ++u) v[u] = b + u < b1 ? __ldcg(&a.loss_part[(size_t)(b + u) * (E + 1) + e]) : 0.f;
#pragma unroll
      for (int u = 0; u < kRB; ++u)
        if (b + u < b1) ps += v[u];
    }
    if (in) pf[g * E + e] = ps;
    float zs = 0.f;
#pragma unroll
    for (int u = 0; u < kRB; ++u)
      if (tid + u * NT < a.nblk) zs += zv[u];
    for (int b = tid + kRB * NT; b < a.nblk; b += kRB * NT) {
      float v[kRB];
#pragma unroll
      for (int u = 0; u < kRB; ++u) {
        const int bb = b + u * NT;
        v[u] = bb < a.nblk ? __ldcg(&a.loss_part[(size_t)bb * (E + 1) + E]) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < kRB; ++u)
        if (b + u * NT < a.nblk) zs += v[u];
    }
    zf[tid] = zs;
  }

  if (!tc) {
    // expert choice: every expert holds exactly ec_count rows
    for (int q = tid; q < E; q += NT) {
      cnt_s[q] = a.ec_count;
      a.cnt_pre[q] = a.ec_count;
    }
    __syncthreads();
  } else {
    int hs = 0;
#pragma unroll
    for (int u = 0; u < kRB; ++u) hs += hv[u];
    for (int c = c0 + kRB; c < c1; c += kRB) {
      int v[kRB];
#pragma unroll
      for (int u = 0; u < kRB; ++u) v[u] = c + u < c1 ? __ldcg(&a.chunk_hist[(size_t)(c + u) * E + e]) : 0;
#pragma unroll
      for (int u = 0; u < kRB; ++u) hs += v[u];
    }
    if (in) gsum[g * E + e] = hs;
    __syncthreads();
    // exclusive scan of the G group sums of each expert: warp w scans experts w, w + NT/32, ...; lane
    // l owns a contiguous run of groups, then a shuffle scan across the lanes (exact integer sums)
    {
      const int warp = tid >> 5, lane = tid & 31;
      const int gpl = (G + 31) / 32;  // groups per lane
      for (int ee = warp; ee < E; ee += NT / 32) {
        const int q0 = min(G, lane * gpl), q1 = min(G, q0 + gpl);
        int local = 0;
        for (int q = q0; q < q1; ++q) local += gsum[q * E + ee];
        int incl = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += v;
        }
        int run = incl - local;
        for (int q = q0; q < q1; ++q) {
          const int v = gsum[q * E + ee];
          gsum[q * E + ee] = run;
          run += v;
        }
        if (lane == 31) {
          cnt_s[ee] = incl;
          a.cnt_pre[ee] = incl;
        }
      }
    }
    __syncthreads();
  }
  if (a.do_dispatch && in) {
    // chunk bases: the first kRB histogram values are still in registers
    int run = gsum[g * E + e];
#pragma unroll
    for (int u = 0; u < kRB; ++u)
      if (c0 + u < c1) {
        a.chunk_base[(size_t)(c0 + u) * E + e] = run;
        run += hv[u];
      }
    for (int c = c0 + kRB; c < c1; c += kRB) {
      int v[kRB];
#pragma unroll
      for (int u = 0; u < kRB; ++u) v[u] = c + u < c1 ? __ldcg(&a.chunk_hist[(size_t)(c + u) * E + e]) : 0;
#pragma unroll
      for (int u = 0; u < kRB; ++u)
        if (c + u < c1) {
          a.chunk_base[(size_t)(c + u) * E + e] = run;
          run += v[u];
        }
    }
  }
  if (a.do_dispatch && tid == 0) {
    int run = 0;
    for (int q = 0; q < E; ++q) {
      long long c = cnt_s[q];
      int kept = (a.cap >= 0 && c > a.cap) ? (int)a.cap : (int)c;
      a.expert_counts[q] = kept;
      a.offsets[q] = run;
      run += kept;
    }
    a.offsets[E] = run;
  }
  if (a.do_losses) {
    __syncthreads();
    for (int w = NT / 2; w >= 32; w >>= 1) {
      if (tid < w) zf[tid] += zf[tid + w];
      __syncthreads();
    }
    if (tid < 32) {
      float z = zf[tid];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
      if (tid == 0) zred[0] = z;
    }
    // P_e: warp w reduces experts w, w + NT/32, ...: lane l sums its contiguous groups, then a fixed
    // shuffle tree (the same order on every run)
    {
      const int warp = tid >> 5, lane = tid & 31;
      const int gpl = (G + 31) / 32;
      for (int ee = warp; ee < E; ee += NT / 32) {
        const int q0 = min(G, lane * gpl), q1 = min(G, q0 + gpl);
        float P = 0.f;
        for (int q = q0; q < q1; ++q) P += pf[q * E + ee];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) P += __shfl_xor_sync(0xffffffffu, P, o);
        // f_e = count_e / (all assignments): T*k, or E*C under expert choice
        const double n_assign = a.ec_count > 0 ? (double)E * a.ec_count : (double)a.T * a.k;
        if (lane == 0) term[ee] = ((double)cnt_s[ee] / n_assign) * ((double)P / (double)a.T);
      }
    }
    __syncthreads();
    if (tid == 0) {
      double sum = 0.0;
      for (int q = 0; q < E; ++q) sum += term[q];
      *a.aux_loss = (float)((double)E * sum);
      *a.z_loss = (float)((double)zred[0] / (double)a.T);
    }
  }
}

// Called by every thread of a block once the block's partial results are written: true in the last
// of `blocks` blocks to get here (the whole grid, or a chunk's CTAs), to which all their writes are then
// visible.  That block also returns the counter to 0 for the next call on the workspace.
__device__ bool last_block_to_finish(unsigned* done, unsigned blocks) {
  __shared__ int s_last;
  __syncthreads();  // the block's writes happen before thread 0's fence below (CTA scope)
  if (threadIdx.x == 0) {
    __threadfence();  // ... and, cumulatively, before its ticket at GPU scope
    s_last = atomicAdd(done, 1u) == blocks - 1;
    if (s_last) {
      __threadfence();  // every earlier block's ticket, and the writes before it, are seen from here on
      atomicExch(done, 0u);
    }
  }
  __syncthreads();
  return s_last != 0;
}

// The reduction fits the last chunk block (256 threads) when each thread reads at most one batch
// of histogram values: k * nblk * E <= kRB * 256.  Larger partials (many experts, long batches) go to
// the one-block reduce kernel of 1024 threads.
bool reduce_fits_router_block(int k, int nblk, int E) {
  return (long long)k * nblk * E <= (long long)kRB * kRouterThreads;
}

// The reduction in the last chunk block of a router (or histogram) grid, when the caller asked for it.
__device__ void fused_reduce_tail(const ReduceArgs& red, unsigned* done) {
  if (done == nullptr) return;
  __shared__ ReduceSmem<kRouterThreads> rs;
  if (last_block_to_finish(done, gridDim.x)) reduce_body<kRouterThreads>(red, rs);
}

// The same reduction spread over blocks of experts, for large k * nblk * E (many experts, long
// batches), where one block would walk long ranges: block b takes experts [b*EB, (b+1)*EB).  Each
// block scans its experts' chunk histograms into chunk bases and totals, sums their P_e into the
// aux terms, and sums one slice of the router blocks' lse^2.  The last block to finish (a ticket on
// a workspace counter) adds the terms and slices in a fixed order and writes the offsets.  Every
// sum has a fixed order, so the results repeat bit for bit.
constexpr int kRedMultiThreads = 256;
struct ReduceMultiSmem {
  int gsum[kRedMultiThreads];
  float pf[kRedMultiThreads];
  float zf[kRedMultiThreads];
  double tv[kRedMultiThreads];  // the last block's copy of the per-expert terms
};

__global__ void __launch_bounds__(kRedMultiThreads) reduce_multi_kernel(ReduceArgs a, int EB) {
  constexpr int NT = kRedMultiThreads;
  __shared__ ReduceMultiSmem sm;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, E = a.E;
  const int C = a.k * a.nblk;
  const int G = NT / EB;  // groups of chunks (EB is a power of 2, at most 16)
  const int g = tid / EB, j = tid % EB;
  const int e = blockIdx.x * EB + j;
  const bool in = e < E;
  const int c0 = (int)((long long)C * g / G), c1 = (int)((long long)C * (g + 1) / G);
  const int b0 = (int)((long long)a.nblk * g / G), b1 = (int)((long long)a.nblk * (g + 1) / G);
  // this block's slice of router blocks for the lse^2 sum
  const int z0 = (int)((long long)a.nblk * blockIdx.x / gridDim.x);
  const int z1 = (int)((long long)a.nblk * (blockIdx.x + 1) / gridDim.x);

  int hv[kRB];
  float pv[kRB];
#pragma unroll
  for (int u = 0; u < kRB; ++u) {
    hv[u] = in && c0 + u < c1 ? __ldcg(&a.chunk_hist[(size_t)(c0 + u) * E + e]) : 0;
    pv[u] = a.do_losses && in && b0 + u < b1 ? __ldcg(&a.loss_part[(size_t)(b0 + u) * (E + 1) + e]) : 0.f;
  }
  int hs = 0;
#pragma unroll
  for (int u = 0; u < kRB; ++u) hs += hv[u];
  for (int c = c0 + kRB; c < c1; c += kRB) {
    int v[kRB];
#pragma unroll
    for (int u = 0; u < kRB; ++u) v[u] = in && c + u < c1 ? __ldcg(&a.chunk_hist[(size_t)(c + u) * E + e]) : 0;
#pragma unroll
    for (int u = 0; u < kRB; ++u) hs += v[u];
  }
  sm.gsum[g * EB + j] = hs;
  if (a.do_losses) {
    float ps = 0.f;
#pragma unroll
    for (int u = 0; u < kRB; ++u)
      if (b0 + u < b1) ps += pv[u];
    for (int b = b0 + kRB; b < b1; b += kRB) {
      float v[kRB];
#pragma unroll
      for (int u = 0; u < kRB; ++u) v[u] = in && b + u < b1 ? __ldcg(&a.loss_part[(size_t)(b + u) * (E + 1) + e]) : 0.f;
#pragma unroll
      for (int u = 0; u < kRB; ++u)
        if (b + u < b1) ps += v[u];
    }
    sm.pf[g * EB + j] = ps;
    float zs = 0.f;
    for (int b = z0 + tid; b < z1; b += NT) zs += __ldcg(&a.loss_part[(size_t)b * (E + 1) + E]);
    sm.zf[tid] = zs;
  }
  __syncthreads();
  // per expert of the block (warp w takes experts w, w + 8, ...): exclusive scan of the G group sums
  // (lane l owns a contiguous run of groups, then a shuffle scan), total, and P_e in the same order
  const double n_assign = (double)a.T * a.k;
  for (int jj = warp; jj < EB; jj += NT / 32) {
    const int ee = blockIdx.x * EB + jj;
    const int gpl = (G + 31) / 32;
    const int q0 = min(G, lane * gpl), q1 = min(G, q0 + gpl);
    int local = 0;
    float P = 0.f;
    for (int q = q0; q < q1; ++q) {
      local += sm.gsum[q * EB + jj];
      if (a.do_losses) P += sm.pf[q * EB + jj];
    }
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) P += __shfl_xor_sync(0xffffffffu, P, o);
    int run = incl - local;
    for (int q = q0; q < q1; ++q) {
      const int v = sm.gsum[q * EB + jj];
      sm.gsum[q * EB + jj] = run;
      run += v;
    }
    if (lane == 31 && ee < E) {
      a.cnt_pre[ee] = incl;
      if (a.do_dispatch) a.expert_counts[ee] = (a.cap >= 0 && incl > a.cap) ? (int)a.cap : incl;
    }
    // every lane holds the full P after the xor tree; lane 31 has the total count
    if (a.do_losses && lane == 31 && ee < E) a.terms[ee] = ((double)incl / n_assign) * ((double)P / (double)a.T);
  }
  __syncthreads();
  if (a.do_dispatch && in) {
    int run = sm.gsum[g * EB + j];
#pragma unroll
    for (int u = 0; u < kRB; ++u)
      if (c0 + u < c1) {
        a.chunk_base[(size_t)(c0 + u) * E + e] = run;
        run += hv[u];
      }
    for (int c = c0 + kRB; c < c1; c += kRB) {
      int v[kRB];
#pragma unroll
      for (int u = 0; u < kRB; ++u) v[u] = c + u < c1 ? __ldcg(&a.chunk_hist[(size_t)(c + u) * E + e]) : 0;
#pragma unroll
      for (int u = 0; u < kRB; ++u)
        if (c + u < c1) {
          a.chunk_base[(size_t)(c + u) * E + e] = run;
          run += v[u];
        }
    }
  }
  if (a.do_losses) {
    for (int w = NT / 2; w >= 32; w >>= 1) {
      if (tid < w) sm.zf[tid] += sm.zf[tid + w];
      __syncthreads();
    }
    if (tid < 32) {
      float z = sm.zf[tid];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
      if (tid == 0) a.zpart[blockIdx.x] = z;
    }
  }
  if (!last_block_to_finish(a.done, gridDim.x)) return;
  // the last block: every thread loads one value of each list (E <= 256, blocks <= 256), then warp 0
  // scans the kept counts into offsets, warp 1 adds the terms and warp 2 the z partials, each lane
  // over 8 consecutive entries and then a fixed shuffle tree
  const int nb = gridDim.x;
  if (tid < E) {
    sm.gsum[tid] = a.do_dispatch ? __ldcg(&a.expert_counts[tid]) : 0;
    sm.tv[tid] = a.do_losses ? __ldcg(&a.terms[tid]) : 0.0;
  } else {
    sm.gsum[tid] = 0;
    sm.tv[tid] = 0.0;
  }
  sm.zf[tid] = (a.do_losses && tid < nb) ? __ldcg(&a.zpart[tid]) : 0.f;
  __syncthreads();
  if (warp == 0 && a.do_dispatch) {
    int v[8], local = 0;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      v[u] = sm.gsum[lane * 8 + u];
      local += v[u];
    }
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    int run = incl - local;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int q = lane * 8 + u;
      if (q <= E) a.offsets[q] = run;  // offsets[E] = the total (the counts past E are 0)
      run += v[u];
    }
    if (lane == 31 && E == kRedMultiThreads) a.offsets[E] = run;  // E = 256: the total is past the lanes' range
  } else if (warp == 1 && a.do_losses) {
    double sum = 0.0;
#pragma unroll
    for (int u = 0; u < 8; ++u) sum += sm.tv[lane * 8 + u];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane == 0) *a.aux_loss = (float)((double)E * sum);
  } else if (warp == 2 && a.do_losses) {
    double z = 0.0;
#pragma unroll
    for (int u = 0; u < 8; ++u) z += (double)sm.zf[lane * 8 + u];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    if (lane == 0) *a.z_loss = (float)(z / (double)a.T);
  }
}

__global__ void __launch_bounds__(1024) reduce_kernel(ReduceArgs a) {
  __shared__ ReduceSmem<1024> sm;
  reduce_body<1024>(a, sm);
}

// The tail below for token choice with E <= 16: L = 8 or 16 lanes per token (lane e of a group holds
// expert e), so a warp takes 32 / L of its 4 tokens at once and every per-token reduction is an
// L-lane shuffle.  Max, sum-exp, lse, p and the top-k come out bitwise as in the 32-lane form (the
// lanes that form holds beyond E add nothing).  Warp w takes the chunk's tokens 4w .. 4w+3.
template <int L>
__device__ void router_finish_narrow(const RouterArgs& a, const float* logits, int epad, float* psum, int* hist,
                                     float* zw, int blk) {
  constexpr int G = 32 / L;  // tokens per pass
  const int E = a.E, T = a.T, k = a.k;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int sub = lane / L, e = lane % L;
  const int t0 = blk * kChunk;
  for (int i = tid; i < k * E; i += kRouterThreads) hist[i] = 0;
  __syncthreads();
  float pacc = 0.f, zacc = 0.f;
#pragma unroll
  for (int pass = 0; pass < 4 / G; ++pass) {
    const int tl = warp * 4 + pass * G + sub;
    const int t = t0 + tl;
    const bool valid = t < T;  // a token past T still takes part in its group's shuffles
    const bool live = e < E;
    const float lv = live ? logits[tl * epad + e] : -INFINITY;
    float m = lv;
#pragma unroll
    for (int o = L / 2; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float ssum = live ? expf(lv - m) : 0.f;
#pragma unroll
    for (int o = L / 2; o > 0; o >>= 1) ssum += __shfl_xor_sync(0xffffffffu, ssum, o);
    const float inv_s = 1.f / ssum;
    const float lse = m + logf(ssum);
    if (valid && live) pacc += expf(lv - m) * inv_s;
    if (valid && e == 0) zacc += lse * lse;
    if (a.logits_out != nullptr && valid && live) a.logits_out[(size_t)t * E + e] = lv;
    // top-k: k rounds of a group arg-max with ties to the lower index
    bool taken = false;
    float psel_sum = 0.f, my_p = 0.f;
    int my_e = -1;
    for (int rr = 0; rr < k; ++rr) {
      float bv = (live && !taken) ? lv : -INFINITY;
      int be = (live && !taken) ? e : 0x7fffffff;
#pragma unroll
      for (int o = L / 2; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oe = __shfl_xor_sync(0xffffffffu, be, o);
        if (ov > bv || (ov == bv && oe < be)) {
          bv = ov;
          be = oe;
        }
      }
      if (be == e) taken = true;
      const float pv = expf(bv - m) * inv_s;
      psel_sum += pv;
      if (e == rr) {
        my_p = pv;
        my_e = be;
      }
    }
    if (valid && e < k) {
      a.topk_idx[(size_t)t * k + e] = my_e;
      a.topk_w[(size_t)t * k + e] = my_p / psel_sum;
      if (a.chunk_hist) atomicAdd(&hist[e * E + my_e], 1);
    }
  }
  // the warp's groups -> lane e (fixed order), then per-warp partials -> smem
#pragma unroll
  for (int o = L; o < 32; o <<= 1) {
    pacc += __shfl_xor_sync(0xffffffffu, pacc, o);
    zacc += __shfl_xor_sync(0xffffffffu, zacc, o);
  }
  if (lane < E) psum[warp * epad + lane] = pacc;
  if (lane == 0) zw[warp] = zacc;
  __syncthreads();
  for (int q = tid; q < E; q += kRouterThreads) {
    float v = 0.f;
    for (int w = 0; w < 8; ++w) v += psum[w * epad + q];
    a.loss_part[(size_t)blk * (E + 1) + q] = v;
  }
  if (tid == 0) {
    float v = 0.f;
    for (int w = 0; w < 8; ++w) v += zw[w];
    a.loss_part[(size_t)blk * (E + 1) + E] = v;
  }
  if (a.chunk_hist) {
    const int nblk = (T + kChunk - 1) / kChunk;
    for (int i = tid; i < k * E; i += kRouterThreads) {
      const int sl = i / E, ex = i % E;
      a.chunk_hist[((size_t)sl * nblk + blk) * E + ex] = hist[i];
    }
  }
  fused_reduce_tail(a.red, a.done);
}

// Softmax, top-k, renormalisation and the block's loss partials from logits[32][epad] in shared
// memory (bias already added).  256 threads: warp w handles the chunk's tokens w, w+8, w+16, w+24.
// psum: [8][epad] floats, hist: [k][E] ints, zw: [8] floats, all shared.
__device__ void router_finish(const RouterArgs& a, const float* logits, int epad, float* psum, int* hist, float* zw,
                              int blk) {
  if (a.scores == nullptr && a.E <= 16) {
    if (a.E <= 8) router_finish_narrow<8>(a, logits, epad, psum, hist, zw, blk);
    else router_finish_narrow<16>(a, logits, epad, psum, hist, zw, blk);
    return;
  }
  const int E = a.E, T = a.T, k = a.k;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t0 = blk * kChunk;
  for (int i = tid; i < k * E; i += kRouterThreads) hist[i] = 0;
  for (int i = tid; i < 8 * epad; i += kRouterThreads) psum[i] = 0.f;
  __syncthreads();

  const int NJ = (E + 31) / 32;  // <= 8
  float pacc[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) pacc[j] = 0.f;
  float zacc = 0.f;
  for (int r = 0; r < 4; ++r) {
    int tl = warp + 8 * r;
    int t = t0 + tl;
    if (t >= T) break;
    float lv[8];
    float m = -INFINITY;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      int e = lane + 32 * j;
      lv[j] = (j < NJ && e < E) ? logits[tl * epad + e] : -INFINITY;
      m = fmaxf(m, lv[j]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float s = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) s += (j < NJ && lane + 32 * j < E) ? expf(lv[j] - m) : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    const float inv_s = 1.f / s;
    const float lse = m + logf(s);
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (j < NJ && lane + 32 * j < E) pacc[j] += expf(lv[j] - m) * inv_s;
    zacc += lse * lse;

    if (a.scores != nullptr) {
      // expert choice: every probability is a combine weight, the logits go out expert-major
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int e = lane + 32 * j;
        if (j < NJ && e < E) {
          a.topk_w[(size_t)t * E + e] = expf(lv[j] - m) * inv_s;
          a.scores[(size_t)e * T + t] = lv[j];
          if (a.logits_out != nullptr) a.logits_out[(size_t)t * E + e] = lv[j];
        }
      }
      if (lane == 0) a.tok_count[t] = 0;
      continue;
    }

    if (a.logits_out != nullptr) {  // training forward: the backward pass recomputes p from these
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int e = lane + 32 * j;
        if (j < NJ && e < E) a.logits_out[(size_t)t * E + e] = lv[j];
      }
    }

    // top-k: k rounds of a warp arg-max with ties to the lower index
    unsigned taken = 0;
    float psel_sum = 0.f;
    float my_p = 0.f;
    int my_e = -1;
    for (int rr = 0; rr < k; ++rr) {
      float bv = -INFINITY;
      int be = 0x7fffffff;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        int e = lane + 32 * j;
        if (j < NJ && e < E && !((taken >> j) & 1u)) {
          if (lv[j] > bv || (lv[j] == bv && e < be)) {
            bv = lv[j];
            be = e;
          }
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        int oe = __shfl_xor_sync(0xffffffffu, be, o);
        if (ov > bv || (ov == bv && oe < be)) {
          bv = ov;
          be = oe;
        }
      }
      if ((be & 31) == lane) taken |= 1u << (be >> 5);
      float pv = expf(bv - m) * inv_s;
      psel_sum += pv;
      if (lane == rr) {
        my_p = pv;
        my_e = be;
      }
    }
    if (lane < k) {
      a.topk_idx[(size_t)t * k + lane] = my_e;
      a.topk_w[(size_t)t * k + lane] = my_p / psel_sum;
      if (a.chunk_hist) atomicAdd(&hist[lane * E + my_e], 1);
    }
  }
  // per-warp partial sums -> smem; then fixed-order sums across warps
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    int e = lane + 32 * j;
    if (j < NJ && e < E) psum[warp * epad + e] = pacc[j];
  }
  if (lane == 0) zw[warp] = zacc;  // every lane holds the same per-warp sum of lse^2
  __syncthreads();
  for (int e = tid; e < E; e += kRouterThreads) {
    float s = 0.f;
    for (int w = 0; w < 8; ++w) s += psum[w * epad + e];
    a.loss_part[(size_t)blk * (E + 1) + e] = s;
  }
  if (tid == 0) {
    float s = 0.f;
    for (int w = 0; w < 8; ++w) s += zw[w];
    a.loss_part[(size_t)blk * (E + 1) + E] = s;
  }
  if (a.chunk_hist) {
    const int nblk = (T + kChunk - 1) / kChunk;  // router chunks
    for (int i = tid; i < k * E; i += kRouterThreads) {
      int s = i / E, e = i % E;
      a.chunk_hist[((size_t)s * nblk + blk) * E + e] = hist[i];
    }
  }
  fused_reduce_tail(a.red, a.done);
}

template <typename TIn>
__global__ void __launch_bounds__(kRouterThreads) router_kernel(RouterArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int E = a.E, H = a.H, T = a.T;
  constexpr int esize = sizeof(TIn);
  const RouterSmem L = router_smem(E, esize);
  const int tid = threadIdx.x;
  const int blk = blockIdx.x;
  const int t0 = blk * kChunk;
  const TIn* x = reinterpret_cast<const TIn*>(a.x);
  const TIn* Wg = reinterpret_cast<const TIn*>(a.Wg);

  const int E4 = L.epad / 4;
  const int P = 8 * E4;                                   // (token quad, expert quad) pairs
  const int KS = P >= kRouterThreads ? 1 : kRouterThreads / P;
  const int PP = P >= kRouterThreads ? (P + kRouterThreads - 1) / kRouterThreads : 1;
  const int ks = (P >= kRouterThreads) ? 0 : tid / P;
  const bool active = (P >= kRouterThreads) || (tid < P * KS);

  const int ntiles = (H + kRouterHC - 1) / kRouterHC;
  const int xchunks_row = kRouterHC * esize / 16;         // 16-byte chunks per x row per stage
  const int wbytes_full = kRouterHC * E * esize;

  auto load_stage = [&](int tile, int stage) {
    unsigned char* xs = smem + stage * (L.xstage + L.wstage);
    unsigned char* ws = xs + L.xstage;
    const int h0 = tile * kRouterHC;
    for (int i = tid; i < kChunk * xchunks_row; i += kRouterThreads) {
      int r = i / xchunks_row, c = i % xchunks_row;
      int t = t0 + r;
      int col = h0 + c * (16 / esize);
      bool ok = (t < T) && (col < H);
      const void* src = ok ? (const void*)(x + (size_t)t * H + col) : (const void*)x;
      cp_async16(xs + r * L.xrow + c * 16, src, ok ? 16 : 0);
    }
    int rows_valid = min(kRouterHC, H - h0);
    int wbytes = rows_valid * E * esize;
    const unsigned char* wsrc = reinterpret_cast<const unsigned char*>(Wg + (size_t)h0 * E);
    for (int i = tid; i < (wbytes_full + 15) / 16; i += kRouterThreads) {
      int off = i * 16;
      int n = wbytes - off;
      n = n < 0 ? 0 : (n > 16 ? 16 : n);
      cp_async16(ws + off, n > 0 ? (const void*)(wsrc + off) : (const void*)Wg, n);
    }
  };

  float acc[2][16];
#pragma unroll
  for (int q = 0; q < 2; ++q)
#pragma unroll
    for (int i = 0; i < 16; ++i) acc[q][i] = 0.f;

#pragma unroll
  for (int s = 0; s < kRouterStages - 1; ++s) {
    if (s < ntiles) load_stage(s, s);
    cp_async_commit();
  }
  for (int tile = 0; tile < ntiles; ++tile) {
    cp_async_wait<kRouterStages - 2>();
    __syncthreads();
    {
      int nt = tile + kRouterStages - 1;
      if (nt < ntiles) load_stage(nt, nt % kRouterStages);
      cp_async_commit();
    }
    const unsigned char* xs = smem + (tile % kRouterStages) * (L.xstage + L.wstage);
    const TIn* wsm = reinterpret_cast<const TIn*>(xs + L.xstage);
    const int hlim = min(kRouterHC, H - tile * kRouterHC);
    if (active) {
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        if (q >= PP) break;
        int p = (P >= kRouterThreads) ? tid + q * kRouterThreads : tid % P;
        if (p >= P) break;
        int tq = p % 8, eq = p / 8;
        for (int hh = ks; hh < hlim; hh += KS) {
          float xv[4], wv[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) xv[j] = to_f32(reinterpret_cast<const TIn*>(xs + (tq + 8 * j) * L.xrow)[hh]);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            int e = eq * 4 + j;
            wv[j] = e < E ? to_f32(wsm[hh * E + e]) : 0.f;
          }
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[q][i * 4 + j] = fmaf(xv[i], wv[j], acc[q][i * 4 + j]);
        }
      }
    }
  }
  cp_async_wait<0>();
  __syncthreads();

  // ---- K-split reduction into logits[32][epad] (+ bias) ----
  float* logits = reinterpret_cast<float*>(smem + L.logits);
  float* red = reinterpret_cast<float*>(smem + L.red);
  const TIn* bg = reinterpret_cast<const TIn*>(a.bg);
  if (KS == 1) {
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      if (q >= PP) break;
      int p = tid + q * kRouterThreads;
      if (p >= P) break;
      int tq = p % 8, eq = p / 8;
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          int e = eq * 4 + j;
          logits[(tq + 8 * i) * L.epad + e] = acc[q][i * 4 + j] + (bg && e < E ? to_f32(bg[e]) : 0.f);
        }
    }
  } else {
    if (active) {
      int p = tid % P;
      int tq = p % 8, eq = p / 8;
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) red[(ks * kChunk + tq + 8 * i) * L.epad + eq * 4 + j] = acc[0][i * 4 + j];
    }
    __syncthreads();
    for (int o = tid; o < kChunk * L.epad; o += kRouterThreads) {
      float s = 0.f;
      for (int q = 0; q < KS; ++q) s += red[q * kChunk * L.epad + o];
      int e = o % L.epad;
      logits[o] = s + (bg && e < E ? to_f32(bg[e]) : 0.f);
    }
  }
  __syncthreads();

  router_finish(a, logits, L.epad, reinterpret_cast<float*>(smem + L.psum), reinterpret_cast<int*>(smem + L.misc),
                reinterpret_cast<float*>(smem + L.misc + 8 * 256 * 4), blockIdx.x);
}

// Streaming router for bf16 with few experts (E <= 16): memory-bound, so the gate weights stay in
// shared memory and each warp streams 4 token rows from HBM with 16-byte loads (lane l reads
// 16-byte chunks l, l+32, ...).  Wg is stored in groups of 8 rows padded by 16 bytes so that the
// 32 lanes, which read rows 8 apart, spread over all banks.
template <int EP>
struct StreamSmem {
  static constexpr int kGroupBytes = 8 * EP * 2 + 16;  // 8 Wg rows of EP bf16 + pad
  static __host__ __device__ int wg_bytes(int H) { return (H / 8) * kGroupBytes; }
  static __host__ __device__ int logits_off(int H) { return (wg_bytes(H) + 15) & ~15; }
  static __host__ __device__ int psum_off(int H) { return logits_off(H) + kChunk * EP * 4; }
  static __host__ __device__ int misc_off(int H) { return psum_off(H) + 8 * EP * 4; }
  static __host__ __device__ int total(int H) { return misc_off(H) + (8 * 256 + 64) * 4; }
};

template <int EP>
__global__ void __launch_bounds__(kRouterThreads) router_stream_kernel(RouterArgs a) {
  using S = StreamSmem<EP>;
  extern __shared__ __align__(16) unsigned char smem[];
  const int E = a.E, H = a.H, T = a.T;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const __nv_bfloat16* Wg = reinterpret_cast<const __nv_bfloat16*>(a.Wg);
  // stage Wg [H][E] -> padded groups of 8 rows x EP columns (zero for e >= E)
  bool staged = false;
  if constexpr (EP >= 8) {
    staged = E == EP;
  }
  if (staged) {
    // whole rows as 16-byte vectors, all loads of a thread issued before its stores
    constexpr int VPR = EP >= 8 ? EP / 8 : 1;  // 16-byte vectors per row
    const uint4* src = reinterpret_cast<const uint4*>(Wg);
    const int nvec = H * VPR;
    for (int i0 = tid; i0 < nvec; i0 += kRouterThreads * 8) {
      uint4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u * kRouterThreads;
        v[u] = i < nvec ? __ldg(src + i) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u * kRouterThreads;
        if (i < nvec) {
          const int h = i / VPR, q = i % VPR;
          *reinterpret_cast<uint4*>(smem + (h >> 3) * S::kGroupBytes + ((h & 7) * EP + 8 * q) * 2) = v[u];
        }
      }
    }
  } else {
    for (int i = tid; i < H * EP; i += kRouterThreads) {
      const int h = i / EP, e = i % EP;
      __nv_bfloat16 v = e < E ? Wg[(size_t)h * E + e] : __float2bfloat16(0.f);
      *reinterpret_cast<__nv_bfloat16*>(smem + (h >> 3) * S::kGroupBytes + ((h & 7) * EP + e) * 2) = v;
    }
  }
  __syncthreads();

  const int tl0 = warp * 4;  // this warp's 4 tokens inside the chunk
  const int t0 = blockIdx.x * kChunk + tl0;
  const int nch = H / 8;  // 16-byte chunks per row
  const uint4* xr[4];
  bool valid[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    valid[i] = t0 + i < T;
    xr[i] = reinterpret_cast<const uint4*>(a.x) + (size_t)(valid[i] ? t0 + i : 0) * nch;
  }
  float acc[4][EP];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int e = 0; e < EP; ++e) acc[i][e] = 0.f;

  constexpr int U = EP <= 8 ? 4 : 2;  // chunks per lane in flight per token
  for (int c0 = lane; c0 < nch; c0 += 32 * U) {
    uint4 xv[U][4];
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int c = c0 + 32 * u;
        xv[u][i] = (valid[i] && c < nch) ? __ldcs(xr[i] + c) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = c0 + 32 * u;
      if (c >= nch) break;
      const unsigned char* grp = smem + c * S::kGroupBytes;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float w[EP];
        if constexpr (EP >= 8) {
#pragma unroll
          for (int q = 0; q < EP / 8; ++q) {  // 16-byte reads: conflict-free with the padded groups
            const uint4 wv = *reinterpret_cast<const uint4*>(grp + (j * EP + 8 * q) * 2);
            const uint32_t ws4[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
            for (int r = 0; r < 4; ++r) {
              const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ws4[r]));
              w[8 * q + 2 * r] = f.x;
              w[8 * q + 2 * r + 1] = f.y;
            }
          }
        } else {
          const uint2 wv = *reinterpret_cast<const uint2*>(grp + j * EP * 2);
          const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wv.x));
          const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wv.y));
          w[0] = lo.x;
          w[1] = lo.y;
          w[2] = hi.x;
          w[3] = hi.y;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t word = (&xv[u][i].x)[j >> 1];
          const float xf = __uint_as_float((j & 1) ? (word & 0xffff0000u) : (word << 16));
#pragma unroll
          for (int e = 0; e < EP; ++e) acc[i][e] = fmaf(xf, w[e], acc[i][e]);
        }
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int e = 0; e < EP; ++e)
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[i][e] += __shfl_xor_sync(0xffffffffu, acc[i][e], o);

  float* logits = reinterpret_cast<float*>(smem + S::logits_off(H));
  if (lane == 0) {
    const __nv_bfloat16* bg = reinterpret_cast<const __nv_bfloat16*>(a.bg);
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int e = 0; e < EP; ++e) logits[(tl0 + i) * EP + e] = acc[i][e] + (bg && e < E ? __bfloat162float(bg[e]) : 0.f);
  }
  __syncthreads();
  router_finish(a, logits, EP, reinterpret_cast<float*>(smem + S::psum_off(H)), reinterpret_cast<int*>(smem + S::misc_off(H)),
                reinterpret_cast<float*>(smem + S::misc_off(H) + 8 * 256 * 4), blockIdx.x);
}

// Tensor-core router for bf16 with E a multiple of 8: the gate GEMM [32 tokens x H] x [H x E] of
// one chunk on mma.sync m16n8k16 (bf16 products are exact in fp32, accumulation in fp32), so the
// kernel stays bound by reading x from HBM for any expert count.  x and Wg tiles of HC columns of
// H stream through a 3-stage cp.async ring (rows padded to an odd number of 16-byte units so the
// ldmatrix row reads hit distinct banks); fragments come from ldmatrix, Wg's (k, n) tile via .trans.
// With fewer than 8 n-tiles the warps split K and their partials are added in a fixed order.
struct MmaRouterPlan {
  int ep8, nt8, ks, hc, xs, ws, stage, logits, red, psum, misc, total;
};

__host__ __device__ inline MmaRouterPlan mma_router_plan(int E, int H) {
  MmaRouterPlan p;
  p.ep8 = (E + 7) & ~7;
  p.nt8 = p.ep8 / 8;
  p.ks = p.nt8 >= 8 ? 1 : 8 / p.nt8;
  int wunits = p.ep8 / 8;
  if ((wunits & 1) == 0) ++wunits;
  p.ws = wunits * 16;
  p.hc = 64;
  for (int hc = 512; hc >= 64; hc >>= 1) {
    const int xs = hc * 2 + 16;
    if (3 * (32 * xs + hc * p.ws) <= 150 * 1024 && hc <= H) {
      p.hc = hc;
      break;
    }
  }
  p.xs = p.hc * 2 + 16;
  p.stage = 32 * p.xs + p.hc * p.ws;
  p.logits = 3 * p.stage;
  p.red = p.logits + 32 * p.ep8 * 4;
  p.psum = p.red + (p.ks > 1 ? p.ks * 32 * p.ep8 * 4 : 0);
  p.misc = p.psum + 8 * p.ep8 * 4;
  p.total = p.misc + (8 * 256 + 64) * 4;
  return p;
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2_trans(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];\n" : "=r"(r0), "=r"(r1) : "r"(addr));
}
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                          uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__global__ void __launch_bounds__(kRouterThreads) router_mma_kernel(RouterArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int E = a.E, H = a.H, T = a.T;
  const MmaRouterPlan P = mma_router_plan(E, H);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t0 = blockIdx.x * kChunk;
  const unsigned char* xg = reinterpret_cast<const unsigned char*>(a.x);
  const unsigned char* wg = reinterpret_cast<const unsigned char*>(a.Wg);
  const int ntiles = (H + P.hc - 1) / P.hc;
  const int xchunks = P.hc / 8;    // 16-byte chunks per x row per stage
  const int wchunks = E / 8;       // 16-byte chunks per Wg row (E % 8 == 0)

  auto load_stage = [&](int tile, int stage) {
    unsigned char* xs = smem + stage * P.stage;
    unsigned char* ws = xs + 32 * P.xs;
    const int h0 = tile * P.hc;
    const int hl = min(P.hc, H - h0);
    for (int i = tid; i < 32 * xchunks; i += kRouterThreads) {
      const int r = i / xchunks, c = i % xchunks;
      const int t = t0 + r;
      const bool ok = t < T && c * 8 < hl;
      const void* src = ok ? (const void*)(xg + ((size_t)t * H + h0 + c * 8) * 2) : (const void*)xg;
      cp_async16(xs + r * P.xs + c * 16, src, ok ? 16 : 0);
    }
    for (int i = tid; i < P.hc * wchunks; i += kRouterThreads) {
      const int r = i / wchunks, c = i % wchunks;
      const bool ok = r < hl;
      const void* src = ok ? (const void*)(wg + ((size_t)(h0 + r) * E + c * 8) * 2) : (const void*)wg;
      cp_async16(ws + r * P.ws + c * 16, src, ok ? 16 : 0);
    }
  };

  // warp's n-tiles and K share
  const int my_ks = P.ks > 1 ? warp / P.nt8 : 0;
  const bool active = P.ks > 1 ? (warp < P.ks * P.nt8) : true;
  float acc[4][2][4];  // [n-tile slot][m-tile][fragment]
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int m = 0; m < 2; ++m)
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[j][m][q] = 0.f;

#pragma unroll
  for (int s = 0; s < 2; ++s) {
    if (s < ntiles) load_stage(s, s);
    cp_async_commit();
  }
  for (int tile = 0; tile < ntiles; ++tile) {
    cp_async_wait<1>();
    __syncthreads();
    if (tile + 2 < ntiles) load_stage(tile + 2, (tile + 2) % 3);
    cp_async_commit();
    const uint32_t xs = (uint32_t)__cvta_generic_to_shared(smem + (tile % 3) * P.stage);
    const uint32_t ws = xs + 32 * P.xs;
    const int ksteps = min(P.hc, H - tile * P.hc) / 16;
    if (active) {
      for (int kk = my_ks; kk < ksteps; kk += P.ks) {
        uint32_t af[2][4];
#pragma unroll
        for (int m = 0; m < 2; ++m) {
          const int row = m * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
          const int col = kk * 16 + (lane >> 4) * 8;
          ldsm_x4(xs + row * P.xs + col * 2, af[m][0], af[m][1], af[m][2], af[m][3]);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int nt = P.ks > 1 ? (j == 0 ? warp % P.nt8 : -1) : warp + 8 * j;
          if (nt < 0 || nt >= P.nt8) continue;
          uint32_t b0, b1;
          const int krow = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
          ldsm_x2_trans(ws + krow * P.ws + nt * 16, b0, b1);
#pragma unroll
          for (int m = 0; m < 2; ++m) mma_16816(acc[j][m], af[m][0], af[m][1], af[m][2], af[m][3], b0, b1);
        }
      }
    }
  }
  cp_async_wait<0>();
  __syncthreads();

  // fragments -> logits[32][ep8] (+ bias); K-split partials added in warp order
  float* logits = reinterpret_cast<float*>(smem + P.logits);
  float* red = reinterpret_cast<float*>(smem + P.red);
  const __nv_bfloat16* bg = reinterpret_cast<const __nv_bfloat16*>(a.bg);
  const int g = lane >> 2, t4 = lane & 3;
  if (active) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int nt = P.ks > 1 ? (j == 0 ? warp % P.nt8 : -1) : warp + 8 * j;
      if (nt < 0 || nt >= P.nt8) continue;
#pragma unroll
      for (int m = 0; m < 2; ++m)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int row = m * 16 + g + (q >= 2 ? 8 : 0);
          const int col = nt * 8 + t4 * 2 + (q & 1);
          if (P.ks > 1) red[(my_ks * 32 + row) * P.ep8 + col] = acc[j][m][q];
          else logits[row * P.ep8 + col] = acc[j][m][q] + (bg && col < E ? __bfloat162float(bg[col]) : 0.f);
        }
    }
  }
  if (P.ks > 1) {
    __syncthreads();
    for (int o = tid; o < 32 * P.ep8; o += kRouterThreads) {
      float v = 0.f;
      for (int q = 0; q < P.ks; ++q) v += red[q * 32 * P.ep8 + o];
      const int col = o % P.ep8;
      logits[o] = v + (bg && col < E ? __bfloat162float(bg[col]) : 0.f);
    }
  }
  __syncthreads();
  router_finish(a, logits, P.ep8, reinterpret_cast<float*>(smem + P.psum), reinterpret_cast<int*>(smem + P.misc),
                reinterpret_cast<float*>(smem + P.misc + 8 * 256 * 4), blockIdx.x);
}

// Register-direct tensor-core router for bf16 with E = 8, 16 or 32 (gate weights resident in
// shared memory): lanes load 16-byte vectors of x straight from HBM, deeply unrolled, and feed
// them to mma.sync m16n8k16 without staging.  Lane (g = lane/4, t = lane%4) loads the 8 columns
// [8t, 8t+8) of a 32-column block for token rows g and g+8; the sum over h does not depend on its
// order, so the fragments use a permuted k (virtual pair {2t, 2t+1} <-> columns {8t, 8t+1},
// {2t+8, 2t+9} <-> {8t+2, 8t+3} in the first MMA; columns 8t+4..8t+7 in the second) and the
// matching Wg^T vector (row e, columns 8t..8t+7) supplies both B fragments.  Warps split H and
// their partial logits are added in warp order.
template <int NT8>
struct DirectSmem {
  static constexpr int E = NT8 * 8;
  static __host__ __device__ int row_bytes(int H) { return H * 2 + 16; }  // Wg^T row, padded
  static __host__ __device__ int red_off(int H) { return E * row_bytes(H); }
  static __host__ __device__ int logits_off(int H) { return red_off(H) + 8 * 32 * E * 4; }
  static __host__ __device__ int psum_off(int H) { return logits_off(H) + 32 * E * 4; }
  static __host__ __device__ int misc_off(int H) { return psum_off(H) + 8 * E * 4; }
  static __host__ __device__ int total(int H) { return misc_off(H) + (8 * 256 + 64) * 4; }
};

template <int NT8>
__global__ void __launch_bounds__(kRouterThreads) router_direct_kernel(RouterArgs a) {
  using S = DirectSmem<NT8>;
  constexpr int E = S::E;
  extern __shared__ __align__(16) unsigned char smem[];
  const int H = a.H, T = a.T;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t4 = lane & 3;
  const int RB = S::row_bytes(H);

  const int t0 = blockIdx.x * kChunk;
  const uint4* xv = reinterpret_cast<const uint4*>(a.x);
  const int rowvec = H / 8;  // 16-byte vectors per token row
  // this lane's token rows: m-tile m, row g (+8)
  int rows[4];
  bool rvalid[4];
#pragma unroll
  for (int m = 0; m < 2; ++m)
#pragma unroll
    for (int hi = 0; hi < 2; ++hi) {
      const int t = t0 + 16 * m + g + 8 * hi;
      rvalid[2 * m + hi] = t < T;
      rows[2 * m + hi] = t < T ? t : 0;
    }
  float acc[2][NT8][4];
#pragma unroll
  for (int m = 0; m < 2; ++m)
#pragma unroll
    for (int n = 0; n < NT8; ++n)
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[m][n][q] = 0.f;

  const int nblk32 = H / 32 / 8;  // 32-column blocks per warp
  const int b0 = warp * nblk32;
  constexpr int U = 4;
  auto load_x = [&](uint4 (&xr)[U][4], int bb) {
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int blk = b0 + bb + u;
        xr[u][r] = (rvalid[r] && bb + u < nblk32) ? __ldcs(xv + (size_t)rows[r] * rowvec + blk * 4 + t4)
                                                  : make_uint4(0, 0, 0, 0);
      }
  };
  uint4 xr[U][4];
  load_x(xr, 0);  // first x loads go out before the gate weights are staged

  // Wg [H][E] -> Wg^T [E][H] (bf16) in shared memory; each thread issues all its loads first
  {
    const uint4* src = reinterpret_cast<const uint4*>(a.Wg);
    const int nvec = H * E / 8;
    for (int i0 = tid; i0 < nvec; i0 += kRouterThreads * 8) {
      uint4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u * kRouterThreads;
        v[u] = i < nvec ? __ldg(src + i) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u * kRouterThreads;
        if (i < nvec) {
          const int h = (i * 8) / E, e0 = (i * 8) % E;
          const uint16_t* pv = reinterpret_cast<const uint16_t*>(&v[u]);
#pragma unroll
          for (int q = 0; q < 8; ++q) *reinterpret_cast<uint16_t*>(smem + (e0 + q) * RB + h * 2) = pv[q];
        }
      }
    }
  }
  __syncthreads();

  auto compute = [&](const uint4 (&xr)[U][4], int bb) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (bb + u >= nblk32) break;
      const int h0 = (b0 + bb + u) * 32;
#pragma unroll
      for (int n = 0; n < NT8; ++n) {
        const uint4 w = *reinterpret_cast<const uint4*>(smem + (n * 8 + g) * RB + (h0 + 8 * t4) * 2);
#pragma unroll
        for (int m = 0; m < 2; ++m) {
          const uint4 xa = xr[u][2 * m], xb = xr[u][2 * m + 1];
          mma_16816(acc[m][n], xa.x, xb.x, xa.y, xb.y, w.x, w.y);
          mma_16816(acc[m][n], xa.z, xb.z, xa.w, xb.w, w.z, w.w);
        }
      }
    }
  };
  // two register groups alternate: the next group's loads are in flight while one is computed
  uint4 xr2[U][4];
  for (int bb = 0; bb < nblk32; bb += 2 * U) {
    if (bb + U < nblk32) load_x(xr2, bb + U);
    compute(xr, bb);
    if (bb + 2 * U < nblk32) load_x(xr, bb + 2 * U);
    if (bb + U < nblk32) compute(xr2, bb + U);
  }
  // per-warp partials -> shared, then a fixed-order sum over warps (+ bias)
  float* red = reinterpret_cast<float*>(smem + S::red_off(H));
#pragma unroll
  for (int m = 0; m < 2; ++m)
#pragma unroll
    for (int n = 0; n < NT8; ++n)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int row = 16 * m + g + (q >= 2 ? 8 : 0);
        const int col = n * 8 + t4 * 2 + (q & 1);
        red[(warp * 32 + row) * E + col] = acc[m][n][q];
      }
  __syncthreads();
  float* logits = reinterpret_cast<float*>(smem + S::logits_off(H));
  const __nv_bfloat16* bg = reinterpret_cast<const __nv_bfloat16*>(a.bg);
  for (int o = tid; o < 32 * E; o += kRouterThreads) {
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) v += red[w * 32 * E + o];
    logits[o] = v + (bg ? __bfloat162float(bg[o % E]) : 0.f);
  }
  __syncthreads();
  router_finish(a, logits, E, reinterpret_cast<float*>(smem + S::psum_off(H)), reinterpret_cast<int*>(smem + S::misc_off(H)),
                reinterpret_cast<float*>(smem + S::misc_off(H) + 8 * 256 * 4), blockIdx.x);
}

// Bulk-copy-streamed tensor-core router for bf16 with E = 8 or 16.  The chunk's 32 token rows and
// the matching rows of the gate stream together through an 8-slot shared-memory ring
// (cp.async.bulk, completing on the slot's mbarrier): stage s brings x[t0..t0+32, s*SC..(s+1)*SC)
// (one copy per token row, one per lane) and Wg[s*SC..(s+1)*SC, :] (contiguous in [H][E]: one copy),
// so each SM keeps up to 8 stages in flight and nothing is staged before the stream starts.
// Warp w owns slot w and the stages w, w + 8, ...; after computing a stage it refills the slot
// with its next one.  Both operands go to mma.sync m16n8k16 through ldmatrix in the natural k order:
//   - A (x rows): ldmatrix.x4 per 16-column step and 16-row m-tile.  Staged rows are SC*2 + 16 bytes
//     apart (16 mod 128), so the 8 rows of each 8x8 matrix fall in 8 different bank groups.
//   - B (the gate rows as stored, [h][E]): for each 8-expert n-tile, one ldmatrix.x4.trans over 32
//     consecutive h (16 bytes of each row) gives the B registers of two 16-column steps.  With E = 8 a
//     row is 16 bytes, so 8 consecutive h fill one 128-byte line and the reads are conflict-free; with
//     E = 16 (32-byte rows) each 8x8 matrix meets a 2-way bank conflict.
// Warps' partial logits are added in warp order.  A ring wait is bounded: one that runs out records
// the error word, the CTA stops streaming, waits (bounded) for its copy in flight and finishes on
// what it has (the results are then invalid and the error word says so).
template <int NT8>
struct TmaRouterSmem {
  static constexpr int E = NT8 * 8;
  static constexpr int SC = NT8 == 1 ? 256 : 128;   // x columns (= gate rows) per stage
  static constexpr int kPitch = SC * 2 + 16;         // bytes per staged x row
  static constexpr int kXBytes = kChunk * kPitch;
  static constexpr int kWBytes = SC * 16;            // one plane's gate rows of a stage
  static constexpr int kStage = kXBytes + NT8 * kWBytes;
  static constexpr int kSlots = 8;                   // one per warp
  // [ring][barriers][psum [8][E] f32][hist [8][E] i32][z [64] f32]; red [8][32][E] and logits
  // [32][E] (f32) reuse the ring once every stage is consumed
  static constexpr int kBarOff = kSlots * kStage;
  static constexpr int kPsumOff = kBarOff + kSlots * 8;
  static constexpr int kHistOff = kPsumOff + 8 * E * 4;
  static constexpr int kZwOff = kHistOff + 8 * E * 4;
  static constexpr int kTotal = kZwOff + 64 * 4;
  static constexpr int kRedOff = 0;
  static constexpr int kLogitsOff = 8 * kChunk * E * 4;
  static_assert(kLogitsOff + kChunk * E * 4 <= kBarOff && kStage % 16 == 0 && kXBytes % 16 == 0, "layout");
};

__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

template <int NT8>
__global__ void __launch_bounds__(kRouterThreads) router_tma_kernel(RouterArgs a) {
  using L = TmaRouterSmem<NT8>;
  constexpr int E = L::E, SC = L::SC, P = L::kPitch;
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ int abort_flag;
  const int H = a.H, T = a.T;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t4 = lane & 3;
  const int t0 = blockIdx.x * kChunk;
  const int rows = min(kChunk, T - t0);
  const int nst = H / SC;  // stages of the chunk
  const uint32_t ring = sm100::smem_u32(smem);
  const uint32_t slot = ring + warp * L::kStage;
  const uint32_t wslot = slot + L::kXBytes;
  const uint32_t bar = ring + L::kBarOff + warp * 8;
  const char* xg = static_cast<const char*>(a.x) + (size_t)t0 * H * 2;
  const char* wg = static_cast<const char*>(a.Wg);

  if (lane == 0) sm100::mbar_init(bar, 1);
  if (tid == 0) abort_flag = 0;
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  __syncthreads();
  // stage s -> this warp's slot: lane r copies token row r (rows past T are not copied; their logits
  // are never used), lanes 32 - NT8 .. 31 copy the gate planes
  auto issue = [&](int s) {
    if (lane == 0) sm100::mbar_arrive_expect_tx(bar, (uint32_t)(rows * SC * 2 + NT8 * L::kWBytes));
    __syncwarp();
    if (lane < rows) bulk_g2s(slot + lane * P, xg + (size_t)lane * H * 2 + (size_t)s * SC * 2, SC * 2, bar);
    // the stage's gate rows [s*SC, (s+1)*SC) x E, contiguous in global memory: one copy
    if (lane == 31) bulk_g2s(wslot, wg + (size_t)s * SC * E * 2, NT8 * L::kWBytes, bar);
  };
  if (warp < nst) issue(warp);

  float acc[2][NT8][4];
#pragma unroll
  for (int m = 0; m < 2; ++m)
#pragma unroll
    for (int n = 0; n < NT8; ++n)
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[m][n][q] = 0.f;
  // ldmatrix row addresses of this lane: matrix i = lane/8, row j = lane%8
  const int mi = lane >> 3, mj = lane & 7;
  // A (x.4, non-transposed): matrices (rows 0-7, k 0-7), (rows 8-15, k 0-7), (rows 0-7, k 8-15),
  // (rows 8-15, k 8-15) of a 16 x 16 block -> a0..a3 of m16n8k16
  const uint32_t a_off = (uint32_t)(((mi & 1) * 8 + mj) * P + (mi >> 1) * 16);
  // B (x.4, transposed): matrix i = gate rows h0 + 8i .. h0 + 8i + 7 of one 8-expert plane -> b0, b1 of
  // the first 16-column step (i = 0, 1) and of the second (i = 2, 3)
  const uint32_t b_off = (uint32_t)((8 * mi + mj) * (E * 2));
  int pending = -1;  // the use of this warp's slot whose copies are in flight and not yet waited for
  int use = 0;       // uses of this warp's slot so far: the barrier phase parity
  for (int s = warp; s < nst; s += 8, ++use) {
    pending = use;
    const bool landed =
        sm100::mbar_wait(bar, (uint32_t)(use & 1), a.wait_limit, &abort_flag, a.status, kDevTimeoutProducer);
    if (!__all_sync(0xffffffffu, landed)) break;  // the whole warp leaves together
    pending = -1;
#pragma unroll 2
    for (int blk = 0; blk < SC / 32; ++blk) {
      uint32_t bq[NT8][4];
#pragma unroll
      for (int n = 0; n < NT8; ++n)
        ldsm_x4_trans(wslot + (uint32_t)(blk * 32 * E * 2) + b_off + n * 16, bq[n][0], bq[n][1], bq[n][2], bq[n][3]);
#pragma unroll
      for (int ks = 0; ks < 2; ++ks) {
        uint32_t af[2][4];
#pragma unroll
        for (int m = 0; m < 2; ++m)
          ldsm_x4(slot + (uint32_t)(m * 16 * P + (blk * 32 + ks * 16) * 2) + a_off, af[m][0], af[m][1], af[m][2], af[m][3]);
#pragma unroll
        for (int n = 0; n < NT8; ++n)
#pragma unroll
          for (int m = 0; m < 2; ++m)
            mma_16816(acc[m][n], af[m][0], af[m][1], af[m][2], af[m][3], bq[n][2 * ks], bq[n][2 * ks + 1]);
      }
    }
    __syncwarp();
    if (s + 8 < nst) {
      asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
      issue(s + 8);
    }
  }
  if (pending >= 0) {  // a wait ran out: let the copies in flight land before the ring is reused
    int dummy = 0;
    sm100::mbar_wait(bar, (uint32_t)(pending & 1), a.wait_limit, &dummy, nullptr, 0);
  }
  __syncthreads();  // every slot consumed: the ring becomes red / logits
  float* red = reinterpret_cast<float*>(smem + L::kRedOff);
#pragma unroll
  for (int m = 0; m < 2; ++m)
#pragma unroll
    for (int n = 0; n < NT8; ++n)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int row = 16 * m + g + (q >= 2 ? 8 : 0);
        const int col = n * 8 + t4 * 2 + (q & 1);
        red[(warp * 32 + row) * E + col] = acc[m][n][q];
      }
  __syncthreads();
  float* logits = reinterpret_cast<float*>(smem + L::kLogitsOff);
  const __nv_bfloat16* bg = reinterpret_cast<const __nv_bfloat16*>(a.bg);
  for (int o = tid; o < 32 * E; o += kRouterThreads) {
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) v += red[w * 32 * E + o];
    logits[o] = v + (bg ? __bfloat162float(bg[o % E]) : 0.f);
  }
  __syncthreads();
  router_finish(a, logits, E, reinterpret_cast<float*>(smem + L::kPsumOff), reinterpret_cast<int*>(smem + L::kHistOff),
                reinterpret_cast<float*>(smem + L::kZwOff), blockIdx.x);
}

// Softmax, top-k, renormalisation and partials of one 32-token chunk from logits that a tensor-core
// GEMM already wrote to global memory ([T,E] fp32, bias included).
__global__ void __launch_bounds__(kRouterThreads) router_logits_finish_kernel(RouterArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int E = a.E;
  float* logits = reinterpret_cast<float*>(smem);  // [32][E]
  float* psum = logits + kChunk * E;                 // [8][E]
  int* misc = reinterpret_cast<int*>(psum + 8 * E);  // [k][E] histogram, then 8 floats
  const int t0 = blockIdx.x * kChunk;
  const int n4 = min(kChunk, a.T - t0) * E / 4;
  const float4* src = reinterpret_cast<const float4*>(a.gemm_logits + (size_t)t0 * E);
  for (int i = threadIdx.x; i < kChunk * E / 4; i += kRouterThreads)
    reinterpret_cast<float4*>(logits)[i] = i < n4 ? src[i] : make_float4(0.f, 0.f, 0.f, 0.f);
  __syncthreads();
  router_finish(a, logits, E, psum, misc, reinterpret_cast<float*>(misc + 8 * 256), blockIdx.x);
}

// Per-chunk, per-slot expert histogram from a given topk_idx (standalone permute).
// An expert index outside [0, E) (from a caller-supplied topk_idx) is not counted; the error word
// records it and moe_get_device_status reports it.
// With done given, the last block also runs the dispatch reduction of red (as the routers do).
__global__ void __launch_bounds__(kRouterThreads) hist_kernel(const int32_t* __restrict__ topk_idx, int T, int E, int k,
                                                          int32_t* __restrict__ chunk_hist, int32_t* status,
                                                          ReduceArgs red, unsigned* done) {
  __shared__ int hist[8 * 256];
  const int blk = blockIdx.x, nblk = gridDim.x, tid = threadIdx.x;
  for (int i = tid; i < k * E; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  if (tid < kChunk * k) {
    int s = tid / kChunk, t = blk * kChunk + (tid % kChunk);
    if (t < T) {
      const int e = topk_idx[(size_t)t * k + s];
      if (e >= 0 && e < E) atomicAdd(&hist[s * E + e], 1);
      else atomicCAS(status, 0, kDevBadIndex);
    }
  }
  __syncthreads();
  for (int i = tid; i < k * E; i += blockDim.x) {
    int s = i / E, e = i % E;
    chunk_hist[((size_t)s * nblk + blk) * E + e] = hist[i];
  }
  fused_reduce_tail(red, done);
}

// Block (chunk b, slot s, column slice z): stable in-chunk ranks by warp match, rows, drop flags and
// row maps (slice 0), the slice of the x row copies into x_perm, and the slice of the clearing of
// the chunk's output rows that falls to this slot (its 32/k rows, so every block stores as much).
__global__ void __launch_bounds__(256) scatter_kernel(ScatterArgs a) {
  __shared__ int rows_s[kChunk];
  __shared__ int tok_s[kChunk];
  const int b = blockIdx.x, s = blockIdx.y, tid = threadIdx.x;
  const int nblk = a.nblk;
  // block z copies and clears only its slice of the columns; every slice ranks the chunk itself (one
  // warp, cheap) and slice 0 writes the row maps
  const bool maps = blockIdx.z == 0;
  if (tid < 32) {
    const int lane = tid;
    const int t = b * kChunk + lane;
    int e = t < a.T ? a.topk_idx[(size_t)t * a.k + s] : -1;
    if (maps && t < a.T && (e < 0 || e >= a.E)) atomicCAS(a.status, 0, kDevBadIndex);  // dropped below, never copied
    const bool valid = t < a.T && e >= 0 && e < a.E;
    if (!valid) e = -1 - lane;  // invalid lanes never match
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rank_local = __popc(peers & ((1u << lane) - 1u));
    int row = -1;
    if (maps && t < a.T && !valid) {
      a.dropped[(size_t)t * a.k + s] = 1;
      a.row_of[(size_t)t * a.k + s] = -1;
    }
    if (valid) {
      const long long rank = (long long)a.chunk_base[((size_t)s * nblk + b) * a.E + e] + rank_local;
      const bool keep = a.cap < 0 || rank < a.cap;
      if (keep) row = a.offsets[e] + (int)rank;
      if (maps) {
        a.dropped[(size_t)t * a.k + s] = keep ? 0 : 1;
        a.row_of[(size_t)t * a.k + s] = row;
        if (keep) {
          a.row_token[row] = t;
          a.row_slot[row] = s;
        }
      }
    }
    rows_s[lane] = row;
    tok_s[lane] = valid ? t : -1;
  }
  __syncthreads();
  if (a.out != nullptr) {
    // this slot's share of the chunk's out rows, inside the batch: the stores go out first and drain
    // while the copies below wait on their loads
    const int r_lo = s * kChunk / (int)gridDim.y;
    const int r_hi = min((s + 1) * kChunk / (int)gridDim.y, a.T - b * kChunk);
    const int ovec = a.H / 4;
    const int o_lo = (int)((long long)ovec * blockIdx.z / gridDim.z);
    const int ow = (int)((long long)ovec * (blockIdx.z + 1) / gridDim.z) - o_lo;
    float4* o = reinterpret_cast<float4*>(a.out) + (size_t)b * kChunk * ovec + o_lo;
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
    const int sr = 256 / ow, sc = 256 % ow;
    int orow = r_lo + tid / ow, oc = tid % ow;
    while (orow < r_hi) {
      o[(size_t)orow * ovec + oc] = z;
      orow += sr;
      oc += sc;
      if (oc >= ow) {
        oc -= ow;
        ++orow;
      }
    }
  }
  const int nvec = a.H * a.esize / 16;  // 16-byte vectors per row
  const uint4* xv = reinterpret_cast<const uint4*>(a.x);
  uint4* pv = reinterpret_cast<uint4*>(a.x_perm);
  // this block's columns [c_lo, c_lo + w) of each row, in 16-byte vectors
  const int c_lo = (int)((long long)nvec * blockIdx.z / gridDim.z);
  const int w = (int)((long long)nvec * (blockIdx.z + 1) / gridDim.z) - c_lo;
  // this thread's (row, vector) walk over the chunk's 32 rows in steps of 256 vectors, with the
  // row / column split kept incrementally (no division per element)
  const int step_r = 256 / w, step_c = 256 % w;
  constexpr int U = 8;  // 16-byte loads in flight per thread
  int r = tid / w, c = tid % w;
  while (r < kChunk) {
    uint4 v[U];
    int dst[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      dst[u] = -1;
      if (r < kChunk) {
        const int row = rows_s[r];
        if (row >= 0) {
          v[u] = xv[(size_t)tok_s[r] * nvec + c_lo + c];
          dst[u] = row * nvec + c_lo + c;  // < T*k*nvec < 2^31 (checked on the host)
        }
      }
      r += step_r;
      c += step_c;
      if (c >= w) {
        c -= w;
        ++r;
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (dst[u] >= 0) pv[dst[u]] = v[u];
  }
}

__global__ void zero_outputs_kernel(int32_t* counts, int E, float* aux, float* z) {
  for (int e = threadIdx.x; e < E; e += blockDim.x) counts[e] = 0;
  if (threadIdx.x == 0) {
    if (aux) *aux = 0.f;
    if (z) *z = 0.f;
  }
}

// out[t] = sum over kept slots (slot order) of w[t,s] * y[row_of[t,s]]; zeros if all dropped.
__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ y, const int32_t* __restrict__ row_of,
                                                      const float* __restrict__ topk_w, int H, int k,
                                                      float* __restrict__ out) {
  const int t = blockIdx.x;
  const int nv = H / 4;
  const float4* yv = reinterpret_cast<const float4*>(y);
  float4* ov = reinterpret_cast<float4*>(out);
  for (int c = threadIdx.x; c < nv; c += blockDim.x) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = 0; s < k; ++s) {
      int row = row_of[(size_t)t * k + s];
      if (row < 0) continue;
      float w = topk_w[(size_t)t * k + s];
      float4 v = yv[(size_t)row * nv + c];
      acc.x = fmaf(w, v.x, acc.x);
      acc.y = fmaf(w, v.y, acc.y);
      acc.z = fmaf(w, v.z, acc.z);
      acc.w = fmaf(w, v.w, acc.w);
    }
    ov[(size_t)t * nv + c] = acc;
  }
}

}  // namespace

// moe_set_kernel_options(MOE_KERNEL_NO_TC_GATE) selects the CUDA-core routers (for comparisons).
bool router_mma_disabled() { return (kernel_options() & MOE_KERNEL_NO_TC_GATE) != 0; }

template <int EP>
cudaError_t launch_stream(const RouterArgs& a, int nblk, cudaStream_t st) {
  const int bytes = StreamSmem<EP>::total(a.H);
  cudaError_t err = ensure_smem_limit(reinterpret_cast<const void*>(router_stream_kernel<EP>), bytes);
  if (err != cudaSuccess) return err;
  router_stream_kernel<EP><<<nblk, kRouterThreads, bytes, st>>>(a);
  return cudaGetLastError();
}

template <int NT8>
cudaError_t launch_tma_router(const RouterArgs& a, int nblk, cudaStream_t st) {
  const int bytes = TmaRouterSmem<NT8>::kTotal;
  cudaError_t err = ensure_smem_limit(reinterpret_cast<const void*>(router_tma_kernel<NT8>), bytes);
  if (err != cudaSuccess) return err;
  router_tma_kernel<NT8><<<nblk, kRouterThreads, bytes, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_router(const RouterArgs& a_in, int dtype, cudaStream_t st, int* launches, bool* reduced) {
  const int nblk = (a_in.T + kChunk - 1) / kChunk;
  // every chunk-by-chunk router below runs the reduction in its last block when done is given and
  // the partials are small enough; the one-GEMM gate (its epilogue covers 128 tokens per tile) does not
  RouterArgs a = a_in;
  if (a.done != nullptr && !reduce_fits_router_block(a.k, nblk, a.E)) a.done = nullptr;
  *reduced = a.done != nullptr;
  // the tcgen05 gate kernels wait on pipeline barriers with a bound, and record a wait that ran out
  // in a device error word: without one (or without a bound) they are not used
  const bool tc_gate_ok = a.status != nullptr && a.wait_limit > 0 && !router_mma_disabled();
  const int sms = a.num_sms > 0 ? a.num_sms : 148;
  // bf16, token choice, E = 64, 128 or 256, and enough 128-token tiles to fill at least half the SMs:
  // one tensor-core GEMM whose epilogue does the whole softmax / top-k / partials tail (the logits
  // never leave the SM).  With fewer tiles each CTA's short k-loop is latency-bound (the Switch shape:
  // 64 tiles of K = 1024 took 36.5 us against 23 us for the two-kernel form below), so the
  // 64-column-tile GEMM + per-chunk tail keeps more SMs streaming.
  if (dtype == MOE_DTYPE_BF16 && a.scores == nullptr && (a.E == 64 || a.E == 128 || a.E == 256) && a.H % 64 == 0 &&
      a.k <= 8 && tc_gate_ok && 2 * ((a.T + 127) / 128) >= sms) {
    ++*launches;
    *reduced = false;
    return launch_gate_router_sm100(a, st);
  }
  // bf16, E a multiple of 64, scratch given: the gate is one dense tensor-core GEMM, then the
  // per-chunk tail (the gate weights are read once per 128-token tile instead of once per chunk)
  if (a.gemm_logits != nullptr && dtype == MOE_DTYPE_BF16 && a.E % 64 == 0 && a.H % 64 == 0 && tc_gate_ok) {
    cudaError_t err = launch_gate_logits_sm100(a.x, a.Wg, a.bg, a.T, a.H, a.E, a.gemm_logits, a.status, a.wait_limit,
                                               a.num_sms > 0 ? a.num_sms : 148, st);
    if (err != cudaSuccess) return err;
    ++*launches;
    const int bytes = (kChunk * a.E + 8 * a.E) * 4 + (8 * 256 + 64) * 4;
    err = ensure_smem_limit(reinterpret_cast<const void*>(router_logits_finish_kernel), bytes);
    if (err != cudaSuccess) return err;
    router_logits_finish_kernel<<<nblk, kRouterThreads, bytes, st>>>(a);
    ++*launches;
    return cudaGetLastError();
  }
  ++*launches;  // every other form is one kernel
  // bf16, E = 8 or 16: x streamed by bulk copies through a shared-memory ring (bounded waits, so an
  // error word and a bound are needed), the gate weights resident
  if (dtype == MOE_DTYPE_BF16 && (a.E == 8 || a.E == 16) && a.status != nullptr && a.wait_limit > 0 &&
      !router_mma_disabled() && (kernel_options() & MOE_KERNEL_NO_TMA_ROUTER) == 0) {
    // (the ring does not depend on H: the gate rows travel with the x stages)
    if (a.E == 8 && a.H % TmaRouterSmem<1>::SC == 0) return launch_tma_router<1>(a, nblk, st);
    if (a.E == 16 && a.H % TmaRouterSmem<2>::SC == 0) return launch_tma_router<2>(a, nblk, st);
  }
  // bf16, E in {8, 16, 32}, Wg^T fits in shared memory: register-direct tensor-core stream over x
  if (dtype == MOE_DTYPE_BF16 && (a.E == 8 || a.E == 16 || a.E == 32) && a.H % 256 == 0 && !router_mma_disabled()) {
    const int bytes = a.E == 8 ? DirectSmem<1>::total(a.H) : (a.E == 16 ? DirectSmem<2>::total(a.H) : DirectSmem<4>::total(a.H));
    if (bytes <= 200 * 1024) {
      const void* kern = a.E == 8 ? reinterpret_cast<const void*>(router_direct_kernel<1>)
                                  : (a.E == 16 ? reinterpret_cast<const void*>(router_direct_kernel<2>)
                                               : reinterpret_cast<const void*>(router_direct_kernel<4>));
      cudaError_t err = ensure_smem_limit(kern, bytes);
      if (err != cudaSuccess) return err;
      if (a.E == 8) router_direct_kernel<1><<<nblk, kRouterThreads, bytes, st>>>(a);
      else if (a.E == 16) router_direct_kernel<2><<<nblk, kRouterThreads, bytes, st>>>(a);
      else router_direct_kernel<4><<<nblk, kRouterThreads, bytes, st>>>(a);
      return cudaGetLastError();
    }
  }
  // bf16 with E a multiple of 8: tensor-core gate tile staged through shared memory
  if (dtype == MOE_DTYPE_BF16 && a.E % 8 == 0 && a.H % 64 == 0 && !router_mma_disabled()) {
    const MmaRouterPlan P = mma_router_plan(a.E, a.H);
    cudaError_t err = ensure_smem_limit(reinterpret_cast<const void*>(router_mma_kernel), P.total);
    if (err != cudaSuccess) return err;
    router_mma_kernel<<<nblk, kRouterThreads, P.total, st>>>(a);
    return cudaGetLastError();
  }
  // other small expert counts: the gate is a weight-resident stream over x (HBM bound)
  if (dtype == MOE_DTYPE_BF16 && a.E <= 16 && a.H % 8 == 0) {
    const int ep = a.E <= 4 ? 4 : (a.E <= 8 ? 8 : 16);
    const int bytes = ep == 4 ? StreamSmem<4>::total(a.H) : (ep == 8 ? StreamSmem<8>::total(a.H) : StreamSmem<16>::total(a.H));
    if (bytes <= 200 * 1024) {
      if (ep == 4) return launch_stream<4>(a, nblk, st);
      if (ep == 8) return launch_stream<8>(a, nblk, st);
      return launch_stream<16>(a, nblk, st);
    }
  }
  const int esize = dtype == MOE_DTYPE_BF16 ? 2 : 4;
  const RouterSmem L = router_smem(a.E, esize);
  cudaError_t err;
  if (dtype == MOE_DTYPE_BF16) {
    err = ensure_smem_limit(reinterpret_cast<const void*>(router_kernel<__nv_bfloat16>), L.total);
    if (err != cudaSuccess) return err;
    router_kernel<__nv_bfloat16><<<nblk, kRouterThreads, L.total, st>>>(a);
  } else {
    err = ensure_smem_limit(reinterpret_cast<const void*>(router_kernel<float>), L.total);
    if (err != cudaSuccess) return err;
    router_kernel<float><<<nblk, kRouterThreads, L.total, st>>>(a);
  }
  return cudaGetLastError();
}

cudaError_t launch_hist(const int32_t* topk_idx, int T, int E, int k, int nblk, int32_t* chunk_hist, int32_t* status,
                        const ReduceArgs& red, unsigned* done, cudaStream_t st, bool* reduced) {
  if (done != nullptr && !reduce_fits_router_block(k, nblk, E)) done = nullptr;
  *reduced = done != nullptr;
  hist_kernel<<<nblk, kRouterThreads, 0, st>>>(topk_idx, T, E, k, chunk_hist, status, red, done);
  return cudaGetLastError();
}

cudaError_t launch_reduce(const ReduceArgs& a, cudaStream_t st) {
  // token choice with more histogram values than one 1024-thread batch: spread over blocks of experts
  const long long C = (long long)a.k * a.nblk;
  if (a.ec_count <= 0 && a.terms != nullptr && a.zpart != nullptr && a.done != nullptr &&
      C * a.E > (long long)kRB * 1024) {
    int EB = 16;  // experts per block: the largest power of 2 (at most 16) with C * EB / 256 <= kRB
    while (EB > 1 && C * EB > (long long)kRB * kRedMultiThreads) EB >>= 1;
    const int nb = (a.E + EB - 1) / EB;
    if (nb <= 256) {
      reduce_multi_kernel<<<nb, kRedMultiThreads, 0, st>>>(a, EB);
      return cudaGetLastError();
    }
  }
  reduce_kernel<<<1, 1024, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_scatter(const ScatterArgs& a, int num_sms, cudaStream_t st) {
  // the rows' columns are split over S blocks per (chunk, slot): 4 where the rows are wide enough,
  // so that each thread has one or two rounds of loads in flight rather than eight (the Mixtral and
  // skewed shapes' scatter measured 7-10% faster than with whole rows), and more, up to 16, while
  // the grid stays within the SMs (decode-sized batches); each slice keeps at least 8 vectors
  // (128 B) of a row and of an out row
  const long long blocks = (long long)a.nblk * a.k;
  int S = 1;
  const int nvec = a.H * a.esize / 16, ovec = a.H / 4;
  while (S < 16 && nvec / (2 * S) >= 8 && ovec / (2 * S) >= 8 && (S < 4 || blocks * 2 * S <= (long long)num_sms))
    S *= 2;
  dim3 grid(a.nblk, a.k, S);
  scatter_kernel<<<grid, 256, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_zero_outputs(int32_t* expert_counts, int E, float* aux, float* z, cudaStream_t st) {
  zero_outputs_kernel<<<1, 256, 0, st>>>(expert_counts, E, aux, z);
  return cudaGetLastError();
}

cudaError_t launch_combine(const float* y, const int32_t* row_of, const float* topk_w, int T, int H, int k, float* out,
                           cudaStream_t st) {
  combine_kernel<<<T, 256, 0, st>>>(y, row_of, topk_w, H, k, out);
  return cudaGetLastError();
}

}  // namespace moe

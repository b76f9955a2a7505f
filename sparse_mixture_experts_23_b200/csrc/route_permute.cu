// Router, loss/dispatch reduction and permutation kernels of the MoE forward pass.
//
// Router ("MoE Training: Mixture of Experts" page, Quick Start MoELayer.forward; Core Concepts 2
// "Routing Mechanisms" and 3 "Load Balancing"):
//   logits = x.Wg + bg, p = softmax(logits), top-k by (logit desc, index asc), w = p_sel / sum p_sel,
//   aux = E * sum_e f_e P_e (f from pre-drop counts / (T*k), P = mean_t p), z = mean_t lse_t^2.
// Dispatch (Core Concepts 4 capacity_factor / drop_tokens; Best Practices 2 capacity tuning):
//   capacity = ceil(CF*T*k/E) or unlimited; assignments ranked per expert in (slot, token) order;
//   rank < capacity kept; the rank is also the row inside the expert's segment.
#include <cuda_bf16.h>
#include <float.h>
#include <math.h>

#include "moe_internal.cuh"

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

template <typename TIn>
__global__ void __launch_bounds__(kRouterThreads) router_kernel(RouterArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int E = a.E, H = a.H, T = a.T, k = a.k;
  constexpr int esize = sizeof(TIn);
  const RouterSmem L = router_smem(E, esize);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
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
          logits[(tq + 8 * i) * L.epad + e] = acc[q][i * 4 + j] + (e < E ? to_f32(bg[e]) : 0.f);
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
      logits[o] = s + (e < E ? to_f32(bg[e]) : 0.f);
    }
  }
  __syncthreads();

  // ---- softmax, top-k, renormalisation, loss partials: warp w handles tokens w, w+8, w+16, w+24 ----
  float* psum = reinterpret_cast<float*>(smem + L.psum);
  int* hist = reinterpret_cast<int*>(smem + L.misc);
  float* zw = reinterpret_cast<float*>(smem + L.misc + 8 * 256 * 4);
  for (int i = tid; i < k * E; i += kRouterThreads) hist[i] = 0;
  for (int i = tid; i < 8 * L.epad; i += kRouterThreads) psum[i] = 0.f;
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
      lv[j] = (j < NJ && e < E) ? logits[tl * L.epad + e] : -INFINITY;
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
    if (j < NJ && e < E) psum[warp * L.epad + e] = pacc[j];
  }
  if (lane == 0) zw[warp] = zacc;  // every lane holds the same per-warp sum of lse^2
  __syncthreads();
  for (int e = tid; e < E; e += kRouterThreads) {
    float s = 0.f;
    for (int w = 0; w < 8; ++w) s += psum[w * L.epad + e];
    a.loss_part[(size_t)blk * (E + 1) + e] = s;
  }
  if (tid == 0) {
    float s = 0.f;
    for (int w = 0; w < 8; ++w) s += zw[w];
    a.loss_part[(size_t)blk * (E + 1) + E] = s;
  }
  if (a.chunk_hist) {
    const int nblk = gridDim.x;
    for (int i = tid; i < k * E; i += kRouterThreads) {
      int s = i / E, e = i % E;
      a.chunk_hist[((size_t)s * nblk + blk) * E + e] = hist[i];
    }
  }
}

// Per-chunk, per-slot expert histogram from a given topk_idx (standalone permute).
__global__ void hist_kernel(const int32_t* __restrict__ topk_idx, int T, int E, int k, int32_t* __restrict__ chunk_hist) {
  __shared__ int hist[8 * 256];
  const int blk = blockIdx.x, nblk = gridDim.x, tid = threadIdx.x;
  for (int i = tid; i < k * E; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  if (tid < kChunk * k) {
    int s = tid / kChunk, t = blk * kChunk + (tid % kChunk);
    if (t < T) atomicAdd(&hist[s * E + topk_idx[(size_t)t * k + s]], 1);
  }
  __syncthreads();
  for (int i = tid; i < k * E; i += blockDim.x) {
    int s = i / E, e = i % E;
    chunk_hist[((size_t)s * nblk + blk) * E + e] = hist[i];
  }
}

// One block: losses from the router partials, per-expert totals, capacity, offsets and the
// exclusive scan of the chunk histograms in (slot, chunk) order.
__global__ void __launch_bounds__(1024) reduce_kernel(ReduceArgs a) {
  __shared__ int gsum[1024];
  __shared__ int cnt_s[256];
  __shared__ double term[256];
  __shared__ float zred[32];
  const int tid = threadIdx.x, E = a.E;
  const int C = a.k * a.nblk;  // chunks in (slot, token-chunk) order
  const int G = 1024 / E;      // groups of chunks
  const int g = tid / E, e = tid % E;
  const bool in = tid < G * E;
  const int c0 = in ? (int)((long long)C * g / G) : 0;
  const int c1 = in ? (int)((long long)C * (g + 1) / G) : 0;

  int s = 0;
  for (int c = c0; c < c1; ++c) s += a.chunk_hist[(size_t)c * E + e];
  if (in) gsum[g * E + e] = s;
  __syncthreads();
  if (tid < E) {
    int run = 0;
    for (int q = 0; q < G; ++q) {
      int v = gsum[q * E + tid];
      gsum[q * E + tid] = run;
      run += v;
    }
    cnt_s[tid] = run;
    a.cnt_pre[tid] = run;
  }
  __syncthreads();
  if (a.do_dispatch && in) {
    int run = gsum[g * E + e];
    for (int c = c0; c < c1; ++c) {
      int v = a.chunk_hist[(size_t)c * E + e];
      a.chunk_base[(size_t)c * E + e] = run;
      run += v;
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
    // P_e: fixed-order sum over router blocks; z: lane-strided then a fixed shuffle tree
    if (tid < E) {
      float P = 0.f;
      for (int b = 0; b < a.nblk; ++b) P += a.loss_part[(size_t)b * (E + 1) + tid];
      term[tid] = ((double)cnt_s[tid] / ((double)a.T * a.k)) * ((double)P / (double)a.T);
    }
    if (tid < 32) {
      float z = 0.f;
      for (int b = tid; b < a.nblk; b += 32) z += a.loss_part[(size_t)b * (E + 1) + E];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
      if (tid == 0) zred[0] = z;
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

// Block (chunk b, slot s): stable in-chunk ranks by warp match, rows, drop flags, row maps,
// the x row copies into x_perm, and (slot 0) clearing of the chunk's output rows.
__global__ void __launch_bounds__(256) scatter_kernel(ScatterArgs a) {
  __shared__ int rows_s[kChunk];
  __shared__ int tok_s[kChunk];
  const int b = blockIdx.x, s = blockIdx.y, tid = threadIdx.x;
  const int nblk = a.nblk;
  if (tid < 32) {
    const int lane = tid;
    const int t = b * kChunk + lane;
    const bool valid = t < a.T;
    const int e = valid ? a.topk_idx[(size_t)t * a.k + s] : -1 - lane;  // invalid lanes never match
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rank_local = __popc(peers & ((1u << lane) - 1u));
    int row = -1;
    if (valid) {
      const long long rank = (long long)a.chunk_base[((size_t)s * nblk + b) * a.E + e] + rank_local;
      const bool keep = a.cap < 0 || rank < a.cap;
      if (keep) row = a.offsets[e] + (int)rank;
      a.dropped[(size_t)t * a.k + s] = keep ? 0 : 1;
      a.row_of[(size_t)t * a.k + s] = row;
      if (keep) {
        a.row_token[row] = t;
        a.row_slot[row] = s;
      }
    }
    rows_s[lane] = row;
    tok_s[lane] = valid ? t : -1;
  }
  __syncthreads();
  const int nvec = a.H * a.esize / 16;  // 16-byte vectors per row
  const uint4* xv = reinterpret_cast<const uint4*>(a.x);
  uint4* pv = reinterpret_cast<uint4*>(a.x_perm);
  const int total = kChunk * nvec;
  for (int i = tid; i < total; i += 256 * 4) {
    uint4 v[4];
    int rr[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      int idx = i + u * 256;
      rr[u] = -1;
      if (idx < total) {
        int r = idx / nvec, c = idx % nvec;
        int row = rows_s[r];
        if (row >= 0) {
          v[u] = xv[(size_t)tok_s[r] * nvec + c];
          rr[u] = idx;
        }
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (rr[u] >= 0) {
        int idx = rr[u];
        int r = idx / nvec, c = idx % nvec;
        pv[(size_t)rows_s[r] * nvec + c] = v[u];
      }
    }
  }
  if (s == 0 && a.out != nullptr) {
    const int ovec = a.H / 4;
    float4* o = reinterpret_cast<float4*>(a.out);
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int i = tid; i < kChunk * ovec; i += 256) {
      int r = i / ovec, c = i % ovec;
      if (tok_s[r] >= 0) o[(size_t)tok_s[r] * ovec + c] = z;
    }
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

cudaError_t launch_router(const RouterArgs& a, int dtype, cudaStream_t st) {
  const int nblk = (a.T + kChunk - 1) / kChunk;
  const int esize = dtype == MOE_DTYPE_BF16 ? 2 : 4;
  const RouterSmem L = router_smem(a.E, esize);
  cudaError_t err;
  if (dtype == MOE_DTYPE_BF16) {
    err = cudaFuncSetAttribute(router_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, L.total);
    if (err != cudaSuccess) return err;
    router_kernel<__nv_bfloat16><<<nblk, kRouterThreads, L.total, st>>>(a);
  } else {
    err = cudaFuncSetAttribute(router_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, L.total);
    if (err != cudaSuccess) return err;
    router_kernel<float><<<nblk, kRouterThreads, L.total, st>>>(a);
  }
  return cudaGetLastError();
}

cudaError_t launch_hist(const int32_t* topk_idx, int T, int E, int k, int nblk, int32_t* chunk_hist, cudaStream_t st) {
  hist_kernel<<<nblk, 256, 0, st>>>(topk_idx, T, E, k, chunk_hist);
  return cudaGetLastError();
}

cudaError_t launch_reduce(const ReduceArgs& a, cudaStream_t st) {
  reduce_kernel<<<1, 1024, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_scatter(const ScatterArgs& a, cudaStream_t st) {
  dim3 grid(a.nblk, a.k);
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

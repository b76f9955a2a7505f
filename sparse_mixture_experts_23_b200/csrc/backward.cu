// Backward pass of the layer, the CUDA-core kernels ("MoE Training: Mixture of Experts" page: the
// layer is trained, and Core Concepts 3 adds the balancing and z losses to the loss).  The
// tensor-core GEMMs of the backward pass live with the forward ones; these kernels move and reduce
// around them.  Notation: row r of the permuted buffers holds token t = row_token[r], slot s =
// row_slot[r], expert e, weight w = topk_w[t,s]; dout = dL/dout.
//
//   bwd_prep_kernel       dperm[r] = bf16(dout[t]), dyperm[r] = bf16(w * dout[t]), dwraw[r] = 0;
//                         clears dx, dWg, dbg, db1 and db2
//   bias_grad_kernel      db2[e] += sum_r w_r dout[t_r] (fp32 dout), db1[e] += sum_r du_r, by row chunks
//   router_bwd_kernel     one warp per token: dw per slot (dwraw + dout . b2[e], 0 when dropped),
//                         renormalisation, softmax, aux- and z-loss terms -> dlogits[t];
//                         dx[t] += Wg dlogits[t]
//   gate_wgrad_kernel     dWg += x^T dlogits and dbg += sum_t dlogits over a chunk of tokens
#include <cuda_bf16.h>
#include <math.h>

#include "moe_internal.cuh"

namespace moe {
namespace {

__device__ __forceinline__ float ld_store(const void* p, size_t i, int f32) {
  return f32 ? reinterpret_cast<const float*>(p)[i] : __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i]);
}

__global__ void __launch_bounds__(256) bwd_prep_kernel(BwdPrepArgs a) {
  const int kept = a.offsets[a.E];
  const int nv = a.H / 4;  // float4 per dout row
  const long long total = (long long)kept * nv;
  const long long stride = (long long)gridDim.x * blockDim.x;
  const float4* dv = reinterpret_cast<const float4*>(a.dout);
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += stride) {
    const int r = (int)(i / nv), c = (int)(i % nv);
    const int t = a.row_token[r];
    const float w = a.topk_w[(size_t)t * a.k + a.row_slot[r]];
    const float4 v = dv[(size_t)t * nv + c];
    if (a.f32) {
      reinterpret_cast<float4*>(a.dperm)[(size_t)r * nv + c] = v;
      reinterpret_cast<float4*>(a.dyperm)[(size_t)r * nv + c] = make_float4(w * v.x, w * v.y, w * v.z, w * v.w);
      continue;
    }
    const __nv_bfloat162 d01 = __floats2bfloat162_rn(v.x, v.y), d23 = __floats2bfloat162_rn(v.z, v.w);
    const __nv_bfloat162 y01 = __floats2bfloat162_rn(w * v.x, w * v.y), y23 = __floats2bfloat162_rn(w * v.z, w * v.w);
    uint2 dd, yy;
    dd.x = *reinterpret_cast<const uint32_t*>(&d01);
    dd.y = *reinterpret_cast<const uint32_t*>(&d23);
    yy.x = *reinterpret_cast<const uint32_t*>(&y01);
    yy.y = *reinterpret_cast<const uint32_t*>(&y23);
    reinterpret_cast<uint2*>(a.dperm)[(size_t)r * nv + c] = dd;
    reinterpret_cast<uint2*>(a.dyperm)[(size_t)r * nv + c] = yy;
  }
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < kept; i += stride) a.dwraw[i] = 0.f;
  const long long nx = (long long)a.T * a.H / 4;
  float4* dx = reinterpret_cast<float4*>(a.dx);
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < nx; i += stride)
    dx[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < (long long)a.H * a.E; i += stride)
    a.dWg[i] = 0.f;
  if (a.dbg)
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < a.E; i += stride) a.dbg[i] = 0.f;
  if (a.db1)
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < (long long)a.E * a.F; i += stride)
      a.db1[i] = 0.f;
  if (a.db2)
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < (long long)a.E * a.H; i += stride)
      a.db2[i] = 0.f;
  if (a.dwmat)
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < (long long)a.T * a.E; i += stride)
      a.dwmat[i] = 0.f;
}

// Bias gradients over 64-row chunks of the permuted rows (a chunk may span experts; rows are
// grouped by expert, so each thread flushes its running sums with one atomic add per expert met):
//   db2[e] += sum_r w_r dout[t_r]   (fp32 dout, two columns per thread)
//   db1[e] += sum_r du[r]           (bf16 du, two columns per thread)
// grid (ceil(rows / 64), ceil(max(H, F) / 512)); the targets are cleared by bwd_prep_kernel.
constexpr int kBgRows = 64;

__global__ void __launch_bounds__(256) bias_grad_kernel(BiasGradArgs a) {
  __shared__ int tok_s[kBgRows];
  __shared__ float w_s[kBgRows];
  __shared__ int e_s[kBgRows];
  __shared__ int offs_s[257];
  const int kept = a.offsets[a.E];
  const int r0 = blockIdx.x * kBgRows;
  if (r0 >= kept) return;
  const int nr = min(kBgRows, kept - r0);
  for (int i = threadIdx.x; i <= a.E; i += 256) offs_s[i] = a.offsets[i];
  __syncthreads();
  if (threadIdx.x < nr) {
    const int r = r0 + threadIdx.x;
    const int t = a.row_token[r];
    tok_s[threadIdx.x] = t;
    w_s[threadIdx.x] = a.topk_w[(size_t)t * a.k + a.row_slot[r]];
    int lo = 0, hi = a.E;  // expert of row r: the last e with offsets[e] <= r
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (offs_s[mid] <= r) lo = mid;
      else hi = mid;
    }
    e_s[threadIdx.x] = lo;
  }
  __syncthreads();
  const int c = 2 * (blockIdx.y * 256 + threadIdx.x);  // first of this thread's two columns
  // The rows are grouped by expert.  Each run of one expert's rows is summed in row order, with the
  // loads of eight rows issued together before their adds, then added into the expert's bias gradient.
  if (a.db2 && c < a.H) {
    for (int i = 0; i < nr;) {
      const int cur = e_s[i];
      int iend = i + 1;
      while (iend < nr && e_s[iend] == cur) ++iend;
      float2 acc = make_float2(0.f, 0.f);
      int j = i;
      for (; j + 8 <= iend; j += 8) {
        float2 d[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) d[q] = *reinterpret_cast<const float2*>(a.dout + (size_t)tok_s[j + q] * a.H + c);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          acc.x = fmaf(w_s[j + q], d[q].x, acc.x);
          acc.y = fmaf(w_s[j + q], d[q].y, acc.y);
        }
      }
      for (; j < iend; ++j) {
        const float2 d = *reinterpret_cast<const float2*>(a.dout + (size_t)tok_s[j] * a.H + c);
        acc.x = fmaf(w_s[j], d.x, acc.x);
        acc.y = fmaf(w_s[j], d.y, acc.y);
      }
      atomicAdd(a.db2 + (size_t)cur * a.H + c, acc.x);
      atomicAdd(a.db2 + (size_t)cur * a.H + c + 1, acc.y);
      i = iend;
    }
  }
  if (a.db1 && c < a.F) {
    const __nv_bfloat162* du = reinterpret_cast<const __nv_bfloat162*>(a.du);
    const float2* duf = reinterpret_cast<const float2*>(a.du);
    auto load = [&](int i) -> float2 {
      const size_t o = ((size_t)(r0 + i) * a.F + c) / 2;
      return a.f32 ? duf[o] : __bfloat1622float2(du[o]);
    };
    for (int i = 0; i < nr;) {
      const int cur = e_s[i];
      int iend = i + 1;
      while (iend < nr && e_s[iend] == cur) ++iend;
      float2 acc = make_float2(0.f, 0.f);
      int j = i;
      for (; j + 8 <= iend; j += 8) {
        float2 v[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) v[q] = load(j + q);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          acc.x += v[q].x;
          acc.y += v[q].y;
        }
      }
      for (; j < iend; ++j) {
        const float2 v = load(j);
        acc.x += v.x;
        acc.y += v.y;
      }
      atomicAdd(a.db1 + (size_t)cur * a.F + c, acc.x);
      atomicAdd(a.db1 + (size_t)cur * a.F + c + 1, acc.y);
      i = iend;
    }
  }
}

// Expert choice: one warp per row r (token t, expert e): dwmat[t,e] = dwraw[r] + dout[t] . b2[e].
__global__ void __launch_bounds__(256) ec_dw_scatter_kernel(EcDwArgs a) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.x * 8 + warp;
  if (r >= a.rows) return;
  const int t = a.row_token[r], e = a.row_slot[r];
  float bdot = 0.f;
  if (a.b2) {
    for (int h = lane; h < a.H; h += 32)
      bdot = fmaf(a.dout[(size_t)t * a.H + h], ld_store(a.b2, (size_t)e * a.H + h, a.f32), bdot);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) bdot += __shfl_xor_sync(0xffffffffu, bdot, o);
  }
  if (lane == 0) a.dwmat[(size_t)t * a.E + e] = a.dwraw[r] + bdot;
}

constexpr int kRbWarps = 8;  // tokens per block

__global__ void __launch_bounds__(32 * kRbWarps) router_bwd_kernel(RouterBwdArgs a) {
  __shared__ float dl_s[kRbWarps][256];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kRbWarps + warp;
  if (t >= a.T) return;  // whole warps leave together; no block-wide barrier follows
  const int E = a.E, k = a.k, H = a.H;
  const int NJ = (E + 31) / 32;
  float lv[8], p[8], dp[8];
  float m = -INFINITY;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int e = lane + 32 * j;
    lv[j] = (j < NJ && e < E) ? a.logits[(size_t)t * E + e] : -INFINITY;
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
  for (int j = 0; j < 8; ++j) p[j] = (j < NJ && lane + 32 * j < E) ? expf(lv[j] - m) * inv_s : 0.f;

  if (a.dwmat != nullptr) {
    // expert choice: the weight of a chosen pair is p itself, so dp = dw (0 for pairs not chosen);
    // the aux term is the same for every expert of a token and cancels in the softmax backward
    float pdp = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = lane + 32 * j;
      dp[j] = (j < NJ && e < E) ? a.dwmat[(size_t)t * E + e] : 0.f;
      if (a.dw_out && j < NJ && e < E) a.dw_out[(size_t)t * E + e] = dp[j];
      pdp += p[j] * dp[j];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) pdp += __shfl_xor_sync(0xffffffffu, pdp, o);
    const float zc = a.d_z * 2.f * lse / (float)a.T;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = lane + 32 * j;
      if (j < NJ && e < E) {
        const float d = p[j] * (dp[j] - pdp) + zc * p[j];
        a.dlogits[(size_t)t * E + e] = d;
        dl_s[warp][e] = d;
      }
    }
  } else {
  // dw per slot: the GEMM's sum_n G h (already in dwraw) plus dout . b2[e]; 0 when dropped
  float dws[8], ws[8];
  int es[8];
  float S = 0.f;
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    dws[q] = ws[q] = 0.f;
    es[q] = 0;
    if (q >= k) continue;
    const int e = a.topk_idx[(size_t)t * k + q];
    es[q] = e;
    float pv = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (j == (e >> 5)) pv = p[j];
    S += __shfl_sync(0xffffffffu, pv, e & 31);
    ws[q] = a.topk_w[(size_t)t * k + q];
    float d = 0.f;
    if (!a.dropped[(size_t)t * k + q]) {
      float bdot = 0.f;
      if (a.b2 && a.f32) {
        for (int h = lane; h < H; h += 32)
          bdot = fmaf(a.dout[(size_t)t * H + h], reinterpret_cast<const float*>(a.b2)[(size_t)e * H + h], bdot);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) bdot += __shfl_xor_sync(0xffffffffu, bdot, o);
      } else if (a.b2) {  // dout[t] . b2[e], four columns per lane per step (H is a multiple of 64)
        const __nv_bfloat16* b2 = reinterpret_cast<const __nv_bfloat16*>(a.b2) + (size_t)e * H;
        for (int h = 4 * lane; h < H; h += 128) {
          const float4 d = *reinterpret_cast<const float4*>(a.dout + (size_t)t * H + h);
          const uint2 bb = *reinterpret_cast<const uint2*>(b2 + h);
          const float2 b01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&bb.x));
          const float2 b23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&bb.y));
          bdot = fmaf(d.x, b01.x, fmaf(d.y, b01.y, fmaf(d.z, b23.x, fmaf(d.w, b23.y, bdot))));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) bdot += __shfl_xor_sync(0xffffffffu, bdot, o);
      }
      d = a.dwraw[a.row_of[(size_t)t * k + q]] + bdot;
    }
    dws[q] = d;
    if (a.dw_out && lane == 0) a.dw_out[(size_t)t * k + q] = d;
  }
  float dww = 0.f;
#pragma unroll
  for (int q = 0; q < 8; ++q) dww += dws[q] * ws[q];
  const float inv_S = 1.f / S;
  const float aux_c = a.d_aux * (float)E / ((float)a.T * (float)a.T * (float)k);  // d_aux E f_e / T = ... * cnt_pre[e]
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int e = lane + 32 * j;
    dp[j] = (j < NJ && e < E) ? aux_c * (float)a.cnt_pre[e] : 0.f;
  }
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const int e = es[q];
    if (q < k && (e & 31) == lane) {
      const float add = (dws[q] - dww) * inv_S;
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (j == (e >> 5)) dp[j] += add;
    }
  }
  float pdp = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) pdp += p[j] * dp[j];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) pdp += __shfl_xor_sync(0xffffffffu, pdp, o);
  const float zc = a.d_z * 2.f * lse / (float)a.T;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int e = lane + 32 * j;
    if (j < NJ && e < E) {
      const float d = p[j] * (dp[j] - pdp) + zc * p[j];
      a.dlogits[(size_t)t * E + e] = d;
      dl_s[warp][e] = d;
    }
  }
  }
  __syncwarp();
  // dx[t] += Wg dlogits[t]: four rows of Wg per lane per step
  if (a.f32) {  // fp32 gate: one row of Wg per lane per step
    const float* wg = reinterpret_cast<const float*>(a.Wg);
    for (int h = lane; h < H; h += 32) {
      float acc = 0.f;
      for (int e = 0; e < E; ++e) acc = fmaf(wg[(size_t)h * E + e], dl_s[warp][e], acc);
      a.dx[(size_t)t * H + h] += acc;
    }
    return;
  }
  const __nv_bfloat16* Wgb = reinterpret_cast<const __nv_bfloat16*>(a.Wg);
  for (int h = 4 * lane; h < H; h += 128) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    if (E % 8 == 0) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4* wrow = reinterpret_cast<const uint4*>(Wgb + (size_t)(h + i) * E);
        for (int e8 = 0; e8 < E / 8; ++e8) {
          const uint4 v = wrow[e8];
          const __nv_bfloat162* w2 = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 f = __bfloat1622float2(w2[q]);
            acc[i] = fmaf(f.x, dl_s[warp][8 * e8 + 2 * q], fmaf(f.y, dl_s[warp][8 * e8 + 2 * q + 1], acc[i]));
          }
        }
      }
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        for (int e = 0; e < E; ++e) acc[i] = fmaf(__bfloat162float(Wgb[(size_t)(h + i) * E + e]), dl_s[warp][e], acc[i]);
    }
    float4* dxp = reinterpret_cast<float4*>(a.dx + (size_t)t * H + h);
    float4 v = *dxp;
    v.x += acc[0];
    v.y += acc[1];
    v.z += acc[2];
    v.w += acc[3];
    *dxp = v;
  }
}

// grid (ceil(H / 512), token chunks): thread j owns columns h, h+1 (h = 2 (256 bx + j)) and, for
// every group of 8 experts, accumulates x[t, h..h+1] dlogits[t, group] over the chunk's tokens
// (dlogits staged in shared memory), then adds into dWg; block column 0 also adds the chunk's sums
// of dlogits into dbg.  dWg and dbg are cleared by bwd_prep_kernel.
constexpr int kGwTokens = 128;

__global__ void __launch_bounds__(256) gate_wgrad_kernel(GateWgradArgs a) {
  __shared__ float dl[kGwTokens][8];
  const int E = a.E, H = a.H;
  const int h = 2 * (blockIdx.x * 256 + threadIdx.x);
  const int t0 = blockIdx.y * kGwTokens, nt = min(kGwTokens, a.T - t0);
  const __nv_bfloat162* x2 = reinterpret_cast<const __nv_bfloat162*>(a.x);
  const float2* xf2 = reinterpret_cast<const float2*>(a.x);
  for (int e0 = 0; e0 < E; e0 += 8) {
    const int ne = min(8, E - e0);
    __syncthreads();
    for (int i = threadIdx.x; i < kGwTokens * 8; i += 256) {
      const int tt = i / 8, q = i % 8;
      dl[tt][q] = (tt < nt && q < ne) ? a.dlogits[(size_t)(t0 + tt) * E + e0 + q] : 0.f;
    }
    __syncthreads();
    if (h < H) {
      float acc0[8], acc1[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) acc0[q] = acc1[q] = 0.f;
#pragma unroll 4
      for (int tt = 0; tt < nt; ++tt) {
        const size_t xo = ((size_t)(t0 + tt) * H + h) / 2;
        const float2 xv = a.f32 ? xf2[xo] : __bfloat1622float2(x2[xo]);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          acc0[q] = fmaf(xv.x, dl[tt][q], acc0[q]);
          acc1[q] = fmaf(xv.y, dl[tt][q], acc1[q]);
        }
      }
#pragma unroll
      for (int q = 0; q < 8; ++q)
        if (q < ne) {
          atomicAdd(a.dWg + (size_t)h * E + e0 + q, acc0[q]);
          atomicAdd(a.dWg + (size_t)(h + 1) * E + e0 + q, acc1[q]);
        }
    }
    if (a.dbg && blockIdx.x == 0 && threadIdx.x < ne) {
      float bsum = 0.f;
      for (int tt = 0; tt < nt; ++tt) bsum += dl[tt][threadIdx.x];
      atomicAdd(a.dbg + e0 + threadIdx.x, bsum);
    }
  }
}

}  // namespace

cudaError_t launch_bwd_prep(const BwdPrepArgs& a, cudaStream_t st) {
  bwd_prep_kernel<<<4 * 148, 256, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_bias_grad(const BiasGradArgs& a, cudaStream_t st) {
  const int cols = a.H > a.F ? a.H : a.F;
  dim3 grid((a.rows_cap + kBgRows - 1) / kBgRows, (cols + 511) / 512);
  bias_grad_kernel<<<grid, 256, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_ec_dw_scatter(const EcDwArgs& a, cudaStream_t st) {
  if (a.rows <= 0) return cudaSuccess;
  ec_dw_scatter_kernel<<<(a.rows + 7) / 8, 256, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_router_bwd(const RouterBwdArgs& a, cudaStream_t st) {
  router_bwd_kernel<<<(a.T + kRbWarps - 1) / kRbWarps, 32 * kRbWarps, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_gate_wgrad(GateWgradArgs a, cudaStream_t st) {
  dim3 grid((a.H + 511) / 512, (a.T + kGwTokens - 1) / kGwTokens);
  gate_wgrad_kernel<<<grid, 256, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace moe

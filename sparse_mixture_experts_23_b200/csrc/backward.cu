// Backward pass of the layer, the CUDA-core kernels ("MoE Training: Mixture of Experts" page: the
// layer is trained, and Core Concepts 3 adds the balancing and z losses to the loss).  The
// tensor-core GEMMs of the backward pass live with the forward ones; these kernels move and reduce
// around them.  Notation: row r of the permuted buffers holds token t = row_token[r], slot s =
// row_slot[r], expert e, weight w = topk_w[t,s]; dout = dL/dout.
//
//   bwd_prep_kernel       dperm[r] = bf16(dout[t]), dyperm[r] = bf16(w * dout[t]), dwraw[r] = 0;
//                         clears dx, dWg and dbg
//   bias_grad_kernel      db2[e] = sum_r w_r dout[t_r] (fp32 dout), db1[e] = sum_r du_r
//   router_bwd_kernel     one warp per token: dw per slot (dwraw + dout . b2[e], 0 when dropped),
//                         renormalisation, softmax, aux- and z-loss terms -> dlogits[t];
//                         dx[t] += Wg dlogits[t]
//   gate_wgrad_kernel     dWg += x^T dlogits and dbg += sum_t dlogits over a chunk of tokens
#include <cuda_bf16.h>
#include <math.h>

#include "moe_internal.cuh"

namespace moe {
namespace {

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
}

// grid (E, ceil(max(H, F/2) / 256)): thread j of block (e, b) owns column 256*b + j of db2[e] and
// the column pair 2*(256*b + j) of db1[e]; rows of the expert's segment are summed in order.
__global__ void __launch_bounds__(256) bias_grad_kernel(BiasGradArgs a) {
  const int e = blockIdx.x;
  const int j = blockIdx.y * 256 + threadIdx.x;
  const int r0 = a.offsets[e], r1 = a.offsets[e + 1];
  if (a.db2 && j < a.H) {
    float acc = 0.f;
    for (int r = r0; r < r1; ++r) {
      const int t = a.row_token[r];
      const float w = a.topk_w[(size_t)t * a.k + a.row_slot[r]];
      acc = fmaf(w, a.dout[(size_t)t * a.H + j], acc);
    }
    a.db2[(size_t)e * a.H + j] = acc;
  }
  if (a.db1 && 2 * j < a.F) {
    float2 acc = make_float2(0.f, 0.f);
    const __nv_bfloat162* du = reinterpret_cast<const __nv_bfloat162*>(a.du);
    for (int r = r0; r < r1; ++r) {
      const float2 v = __bfloat1622float2(du[(size_t)r * (a.F / 2) + j]);
      acc.x += v.x;
      acc.y += v.y;
    }
    a.db1[(size_t)e * a.F + 2 * j] = acc.x;
    a.db1[(size_t)e * a.F + 2 * j + 1] = acc.y;
  }
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
      if (a.b2) {
        const __nv_bfloat16* b2 = a.b2 + (size_t)e * H;
        for (int h = lane; h < H; h += 32) bdot = fmaf(a.dout[(size_t)t * H + h], __bfloat162float(b2[h]), bdot);
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
  __syncwarp();
  // dx[t] += Wg dlogits[t]
  for (int h = lane; h < H; h += 32) {
    const __nv_bfloat16* wrow = a.Wg + (size_t)h * E;
    float acc = 0.f;
    for (int e = 0; e < E; ++e) acc = fmaf(__bfloat162float(wrow[e]), dl_s[warp][e], acc);
    a.dx[(size_t)t * H + h] += acc;
  }
}

// grid (ceil(H / 256), token chunks): thread j owns h = 256*bx + j and accumulates x[t,h] dlogits[t,:]
// over the chunk's tokens (staged in shared memory), then adds into dWg; block column 0 also adds
// the chunk's dlogits sums into dbg.
constexpr int kGwTokens = 32;

__global__ void __launch_bounds__(256) gate_wgrad_kernel(GateWgradArgs a) {
  __shared__ float dl[kGwTokens][32];
  __shared__ __nv_bfloat16 xs[kGwTokens][256];
  const int E = a.E, H = a.H;
  const int h = blockIdx.x * 256 + threadIdx.x;
  const int tc0 = blockIdx.y * a.chunk, tc1 = min(a.T, tc0 + a.chunk);
  for (int e0 = 0; e0 < E; e0 += 32) {
    const int ne = min(32, E - e0);
    float acc[32];
#pragma unroll
    for (int q = 0; q < 32; ++q) acc[q] = 0.f;
    float bsum = 0.f;
    for (int t0 = tc0; t0 < tc1; t0 += kGwTokens) {
      const int nt = min(kGwTokens, tc1 - t0);
      __syncthreads();
      for (int i = threadIdx.x; i < nt * ne; i += 256) {
        const int tt = i / ne, q = i % ne;
        dl[tt][q] = a.dlogits[(size_t)(t0 + tt) * E + e0 + q];
      }
      for (int tt = 0; tt < nt; ++tt) xs[tt][threadIdx.x] = h < H ? a.x[(size_t)(t0 + tt) * H + h] : __float2bfloat16(0.f);
      __syncthreads();
      if (h < H) {
        for (int tt = 0; tt < nt; ++tt) {
          const float xv = __bfloat162float(xs[tt][threadIdx.x]);
#pragma unroll
          for (int q = 0; q < 32; ++q)
            if (q < ne) acc[q] = fmaf(xv, dl[tt][q], acc[q]);
        }
      }
      if (a.dbg && blockIdx.x == 0 && threadIdx.x < ne)
        for (int tt = 0; tt < nt; ++tt) bsum += dl[tt][threadIdx.x];
    }
    if (h < H) {
#pragma unroll
      for (int q = 0; q < 32; ++q)
        if (q < ne) atomicAdd(a.dWg + (size_t)h * E + e0 + q, acc[q]);
    }
    if (a.dbg && blockIdx.x == 0 && threadIdx.x < ne) atomicAdd(a.dbg + e0 + threadIdx.x, bsum);
  }
}

}  // namespace

cudaError_t launch_bwd_prep(const BwdPrepArgs& a, cudaStream_t st) {
  bwd_prep_kernel<<<4 * 148, 256, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_bias_grad(const BiasGradArgs& a, cudaStream_t st) {
  const int cols = a.H > a.F / 2 ? a.H : a.F / 2;
  dim3 grid(a.E, (cols + 255) / 256);
  bias_grad_kernel<<<grid, 256, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_router_bwd(const RouterBwdArgs& a, cudaStream_t st) {
  router_bwd_kernel<<<(a.T + kRbWarps - 1) / kRbWarps, 32 * kRbWarps, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_gate_wgrad(GateWgradArgs a, cudaStream_t st) {
  // enough token chunks to fill the GPU about twice, given ceil(H / 256) column blocks
  const int hb = (a.H + 255) / 256;
  int chunks = (2 * 148 + hb - 1) / hb;
  if (chunks < 1) chunks = 1;
  a.chunk = (a.T + chunks - 1) / chunks;
  if (a.chunk < kGwTokens) a.chunk = kGwTokens;
  chunks = (a.T + a.chunk - 1) / a.chunk;
  dim3 grid(hb, chunks);
  gate_wgrad_kernel<<<grid, 256, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace moe

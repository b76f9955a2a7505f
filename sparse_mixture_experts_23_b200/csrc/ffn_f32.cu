// fp32 expert FFN on CUDA cores (the fp32 storage path; tensor cores are used for bf16).
//
// Expert ("MoE Training: Mixture of Experts" page, Quick Start: Linear(H, 4H) -> GELU ->
// Linear(4H, H)) applied to every expert segment of the permuted rows:
//   GEMM1: h[r,:] = act(x_perm[r,:] . W1[e] + b1[e])   (GELU exact erf form, or SiLU for the
//          Mixtral block's experts; a null b1 / b2 is a zero bias)
//   GEMM2: fused   out[token(r),:] += w(r) * (h[r,:] . W2[e] + b2[e])
//          unfused y[r,:]           =          h[r,:] . W2[e] + b2[e]
// One block computes a 64x64 tile of one expert segment; the tile -> (expert, row block) map
// comes from the segment offsets written by the permute stage.
#include <math.h>

#include "moe_internal.cuh"

namespace moe {

namespace {

constexpr int BM = 64, BN = 64, BK = 16;

enum { EPI_GELU = 0, EPI_COMBINE = 1, EPI_STORE_Y = 2, EPI_SILU = 3 };

__device__ __forceinline__ float gelu_erf(float u) { return 0.5f * u * (1.f + erff(u * 0.70710678118654752f)); }
// u * sigmoid(u) with the accurate exponential and an IEEE divide (fp32 path)
__device__ __forceinline__ float silu(float u) { return u / (1.f + expf(-u)); }

template <int EPI>
__global__ void __launch_bounds__(256) ffn_f32_kernel(FfnArgs a, const float* __restrict__ A, const float* __restrict__ W,
                                                      const float* __restrict__ bias, int N, int K) {
  __shared__ int mt_prefix[257];
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][BN + 4];
  const int E = a.E, tid = threadIdx.x;
  if (tid == 0) {
    int run = 0;
    for (int e = 0; e < E; ++e) {
      mt_prefix[e] = run;
      run += (a.offsets[e + 1] - a.offsets[e] + BM - 1) / BM;
    }
    mt_prefix[E] = run;
  }
  __syncthreads();
  const int mt = blockIdx.x;
  if (mt >= mt_prefix[E]) return;
  int e = 0;
  while (mt_prefix[e + 1] <= mt) ++e;
  const int seg0 = a.offsets[e], cnt = a.offsets[e + 1] - seg0;
  const int m0 = (mt - mt_prefix[e]) * BM;
  const int rows = min(BM, cnt - m0);
  const int n0 = blockIdx.y * BN;
  const float* Wexp = W + (size_t)e * K * N;

  const int tx = tid % 16, ty = tid / 16;  // 16 x 16 threads, 4x4 outputs each
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

  for (int k0 = 0; k0 < K; k0 += BK) {
    for (int i = tid; i < BM * BK; i += 256) {
      int r = i / BK, kk = i % BK;
      float v = 0.f;
      if (r < rows && k0 + kk < K) v = A[(size_t)(seg0 + m0 + r) * K + k0 + kk];
      As[kk][r] = v;
    }
    for (int i = tid; i < BK * BN; i += 256) {
      int kk = i / BN, c = i % BN;
      float v = 0.f;
      if (k0 + kk < K && n0 + c < N) v = Wexp[(size_t)(k0 + kk) * N + n0 + c];
      Bs[kk][c] = v;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float av[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) av[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) bv[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }

#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int r = ty * 4 + i;
    if (r >= rows) continue;
    int grow = seg0 + m0 + r;
    float w = 0.f;
    int tok = 0;
    if (EPI == EPI_COMBINE) {
      tok = a.row_token[grow];
      w = a.topk_w[(size_t)tok * a.k + a.row_slot[grow]];
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      int n = n0 + tx * 4 + j;
      if (n >= N) continue;
      float v = acc[i][j] + (bias ? bias[(size_t)e * N + n] : 0.f);
      if (EPI == EPI_GELU || EPI == EPI_SILU) {
        reinterpret_cast<float*>(a.h)[(size_t)grow * N + n] = EPI == EPI_GELU ? gelu_erf(v) : silu(v);
        if (a.u_out) reinterpret_cast<float*>(a.u_out)[(size_t)grow * N + n] = v;  // training forward
      } else if (EPI == EPI_COMBINE) {
        atomicAdd(&a.out[(size_t)tok * N + n], w * v);
      } else {
        a.y[(size_t)grow * N + n] = v;
      }
    }
  }
}

}  // namespace

cudaError_t launch_ffn_f32(const FfnArgs& a, cudaStream_t st, int* launches) {
  // upper bound on sum_e ceil(cnt_e / BM): ceil(rows / BM) + E
  const int mt_max = (a.rows_cap + BM - 1) / BM + a.E;
  {
    dim3 grid(mt_max, (a.F + BN - 1) / BN);
    auto kern = a.act == MOE_ACT_SILU ? ffn_f32_kernel<EPI_SILU> : ffn_f32_kernel<EPI_GELU>;
    kern<<<grid, 256, 0, st>>>(a, reinterpret_cast<const float*>(a.x_perm), reinterpret_cast<const float*>(a.W1),
                               reinterpret_cast<const float*>(a.b1), a.F, a.H);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    ++*launches;
  }
  {
    dim3 grid(mt_max, (a.H + BN - 1) / BN);
    const float* hh = reinterpret_cast<const float*>(a.h);
    if (a.fuse_combine)
      ffn_f32_kernel<EPI_COMBINE><<<grid, 256, 0, st>>>(a, hh, reinterpret_cast<const float*>(a.W2),
                                                        reinterpret_cast<const float*>(a.b2), a.H, a.F);
    else
      ffn_f32_kernel<EPI_STORE_Y><<<grid, 256, 0, st>>>(a, hh, reinterpret_cast<const float*>(a.W2),
                                                        reinterpret_cast<const float*>(a.b2), a.H, a.F);
    ++*launches;
  }
  return cudaGetLastError();
}

}  // namespace moe

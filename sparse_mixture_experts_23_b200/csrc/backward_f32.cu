// Backward pass for fp32 storage on CUDA cores (the bf16 path uses the tensor cores).  Same
// definitions as the bf16 backward ("MoE Training: Mixture of Experts" page; the chain rule through
// the forward pass), with every intermediate kept in fp32:
//   dgrad_f32_kernel<EPI_DGRAD_*>   G = dperm . W2[e]^T; dw[r] += G . h; du = w G act'(u)
//   dgrad_f32_kernel<EPI_SCATTER>   dx[t] += du . W1[e]^T
//   wgrad_f32_kernel                dW[e] = A_e^T . B_e over the expert's rows
// One block computes a 64 x 64 tile; weights W[e] are read in place ([E][N][K] for the data
// gradients, k contiguous).
#include <math.h>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int BM = 64, BN = 64, BK = 16;
enum { EPI_DGRAD_GELU = 0, EPI_DGRAD_SILU = 1, EPI_SCATTER = 2 };

__device__ __forceinline__ float gelu_grad_f32(float u) {
  return 0.5f * (1.f + erff(u * 0.70710678118654752f)) + u * 0.3989422804014327f * expf(-0.5f * u * u);
}
__device__ __forceinline__ float silu_grad_f32(float u) {
  const float s = 1.f / (1.f + expf(-u));
  return s * (1.f + u * (1.f - s));
}

struct DgradF32Args {
  const int32_t* offsets;
  int E, N, K, k;
  const float* A;        // [rows, K]
  const float* W;        // [E, N, K]
  const int32_t* row_token;
  const int32_t* row_slot;
  const float* topk_w;   // [T, k] (weights of the rows)
  const float* h_in;     // [rows, N] (dgrad of W2)
  const float* u_in;     // [rows, N]
  float* du_out;         // [rows, N]
  float* dwraw;          // [rows]
  float* dx;             // [T, N] (scatter)
};

template <int EPI>
__global__ void __launch_bounds__(256) dgrad_f32_kernel(DgradF32Args a) {
  __shared__ int mt_prefix[257];
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][BN + 4];
  const int E = a.E, tid = threadIdx.x, N = a.N, K = a.K;
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
  const float* Wexp = a.W + (size_t)e * N * K;
  const int tx = tid % 16, ty = tid / 16;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  for (int k0 = 0; k0 < K; k0 += BK) {
    for (int i = tid; i < BM * BK; i += 256) {
      const int r = i / BK, kk = i % BK;
      As[kk][r] = (r < rows && k0 + kk < K) ? a.A[(size_t)(seg0 + m0 + r) * K + k0 + kk] : 0.f;
    }
    for (int i = tid; i < BN * BK; i += 256) {
      const int c = i / BK, kk = i % BK;  // k fastest: W[e][n][k] is k contiguous
      Bs[kk][c] = (n0 + c < N && k0 + kk < K) ? Wexp[(size_t)(n0 + c) * K + k0 + kk] : 0.f;
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
    const int r = ty * 4 + i;
    if (r >= rows) continue;
    const int grow = seg0 + m0 + r;
    const int tok = a.row_token[grow];
    if (EPI == EPI_SCATTER) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int n = n0 + tx * 4 + j;
        if (n < N) atomicAdd(&a.dx[(size_t)tok * N + n], acc[i][j]);
      }
    } else {
      const float w = a.topk_w[(size_t)tok * a.k + a.row_slot[grow]];
      float dw = 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int n = n0 + tx * 4 + j;
        if (n >= N) continue;
        const size_t o = (size_t)grow * N + n;
        dw = fmaf(acc[i][j], a.h_in[o], dw);
        const float ug = EPI == EPI_DGRAD_SILU ? silu_grad_f32(a.u_in[o]) : gelu_grad_f32(a.u_in[o]);
        a.du_out[o] = w * acc[i][j] * ug;
      }
      atomicAdd(&a.dwraw[grow], dw);
    }
  }
}

// dW[e][m][n] = sum over the expert's rows r of A[r][m] B[r][n]; grid (tiles of one expert, E).
__global__ void __launch_bounds__(256) wgrad_f32_kernel(const int32_t* __restrict__ offsets, int M, int N,
                                                        const float* __restrict__ A, const float* __restrict__ B,
                                                        float* __restrict__ out) {
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][BN + 4];
  const int e = blockIdx.y, tid = threadIdx.x;
  const int MT = (M + BM - 1) / BM;
  const int m0 = (blockIdx.x % MT) * BM, n0 = (blockIdx.x / MT) * BN;
  const int r0 = offsets[e], cnt = offsets[e + 1] - r0;
  const int tx = tid % 16, ty = tid / 16;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  for (int k0 = 0; k0 < cnt; k0 += BK) {
    for (int i = tid; i < BK * BM; i += 256) {
      const int kk = i / BM, mm = i % BM;
      As[kk][mm] = (k0 + kk < cnt && m0 + mm < M) ? A[(size_t)(r0 + k0 + kk) * M + m0 + mm] : 0.f;
    }
    for (int i = tid; i < BK * BN; i += 256) {
      const int kk = i / BN, nn = i % BN;
      Bs[kk][nn] = (k0 + kk < cnt && n0 + nn < N) ? B[(size_t)(r0 + k0 + kk) * N + n0 + nn] : 0.f;
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
    const int m = m0 + ty * 4 + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n < N) out[((size_t)e * M + m) * N + n] = acc[i][j];
    }
  }
}

}  // namespace

cudaError_t launch_bwd_gemms_f32(const BwdGemmArgs& a, cudaStream_t st, int* launches) {
  const int mt_max = (a.rows_cap + BM - 1) / BM + a.E;  // upper bound on sum_e ceil(cnt_e / BM)
  DgradF32Args d{};
  d.offsets = a.offsets;
  d.E = a.E;
  d.k = a.k;
  d.row_token = a.row_token;
  d.row_slot = a.row_slot;
  d.topk_w = a.topk_w;
  // G = dperm . W2[e]^T (W2 stored [E][F][H]: N = F, K = H) -> du, dw partials
  d.N = a.F;
  d.K = a.H;
  d.A = reinterpret_cast<const float*>(a.dperm);
  d.W = reinterpret_cast<const float*>(a.W2);
  d.h_in = reinterpret_cast<const float*>(a.h);
  d.u_in = reinterpret_cast<const float*>(a.u);
  d.du_out = reinterpret_cast<float*>(a.du);
  d.dwraw = a.dwraw;
  {
    dim3 grid(mt_max, (a.F + BN - 1) / BN);
    if (a.act == MOE_ACT_SILU) dgrad_f32_kernel<EPI_DGRAD_SILU><<<grid, 256, 0, st>>>(d);
    else dgrad_f32_kernel<EPI_DGRAD_GELU><<<grid, 256, 0, st>>>(d);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    ++*launches;
  }
  // dx[t] += du . W1[e]^T (W1 stored [E][H][F]: N = H, K = F)
  d.N = a.H;
  d.K = a.F;
  d.A = reinterpret_cast<const float*>(a.du);
  d.W = reinterpret_cast<const float*>(a.W1);
  d.dx = a.dx;
  {
    dim3 grid(mt_max, (a.H + BN - 1) / BN);
    dgrad_f32_kernel<EPI_SCATTER><<<grid, 256, 0, st>>>(d);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    ++*launches;
  }
  // dW2[e] = h_e^T . dyperm_e (F x H); dW1[e] = x_perm_e^T . du_e (H x F)
  {
    dim3 grid(((a.F + BM - 1) / BM) * ((a.H + BN - 1) / BN), a.E);
    wgrad_f32_kernel<<<grid, 256, 0, st>>>(a.offsets, a.F, a.H, reinterpret_cast<const float*>(a.h),
                                           reinterpret_cast<const float*>(a.dyperm), a.dW2);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    ++*launches;
  }
  {
    dim3 grid(((a.H + BM - 1) / BM) * ((a.F + BN - 1) / BN), a.E);
    wgrad_f32_kernel<<<grid, 256, 0, st>>>(a.offsets, a.H, a.F, reinterpret_cast<const float*>(a.x_perm),
                                           reinterpret_cast<const float*>(a.du), a.dW1);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    ++*launches;
  }
  return cudaSuccess;
}

}  // namespace moe

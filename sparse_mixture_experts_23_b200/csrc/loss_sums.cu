// Additive loss sums of one batch and the losses from (possibly all-reduced) sums -- for data-
// parallel replicas that want the losses of the whole batch ("MoE Training" page, Core Concepts 3).
//   aux = E * sum_e (cnt_e / sum cnt) * (Psum_e / T),   z = Zsum / T
// Layout of the sums: [cnt_e (E)][Psum_e (E)][Zsum][T].
#include "moe_internal.cuh"

namespace moe {
namespace {

// One block.  Thread c sums column c of the router's per-chunk partials (Psum_e for c < E, Zsum
// for c = E) over the chunks in order, in double; the pre-drop counts come from the dispatch
// reduction.
__global__ void loss_sums_kernel(const float* loss_part, const int32_t* cnt_pre, int nblk, int E, int T, float* sums) {
  for (int c = threadIdx.x; c <= E; c += blockDim.x) {
    double s = 0.0;
    for (int b = 0; b < nblk; ++b) s += (double)loss_part[(size_t)b * (E + 1) + c];
    sums[c < E ? E + c : 2 * E] = (float)s;
  }
  for (int e = threadIdx.x; e < E; e += blockDim.x) sums[e] = T > 0 ? (float)cnt_pre[e] : 0.f;
  if (threadIdx.x == 0) sums[2 * E + 1] = (float)T;
}

// One thread, fixed order, double: the two losses from the sums.
__global__ void losses_from_sums_kernel(const float* sums, int E, float* aux, float* z) {
  if (threadIdx.x != 0) return;
  double n = 0.0;
  for (int e = 0; e < E; ++e) n += (double)sums[e];
  const double T = (double)sums[2 * E + 1];
  if (!(T > 0.0) || !(n > 0.0)) {
    *aux = 0.f;
    *z = 0.f;
    return;
  }
  double a = 0.0;
  for (int e = 0; e < E; ++e) a += ((double)sums[e] / n) * ((double)sums[E + e] / T);
  *aux = (float)((double)E * a);
  *z = (float)((double)sums[2 * E] / T);
}

}  // namespace

cudaError_t launch_loss_sums(const float* loss_part, const int32_t* cnt_pre, int nblk, int E, int T, float* sums,
                             cudaStream_t st) {
  loss_sums_kernel<<<1, 288, 0, st>>>(loss_part, cnt_pre, nblk, E, T, sums);
  return cudaGetLastError();
}

cudaError_t launch_losses_from_sums(const float* sums, int E, float* aux, float* z, cudaStream_t st) {
  losses_from_sums_kernel<<<1, 32, 0, st>>>(sums, E, aux, z);
  return cudaGetLastError();
}

}  // namespace moe

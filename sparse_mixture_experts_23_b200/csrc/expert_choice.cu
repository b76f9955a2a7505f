// Expert-choice routing ("MoE Training: Mixture of Experts" page, Core Concepts 2, "Expert Choice
// Routing"): the router's logits are read per expert and every expert takes the C tokens with the
// largest logits (ties to the lower token index), so every expert holds exactly C rows.
//
//   ec_select_kernel   one 1024-thread block per expert: radix select of the C-th largest logit
//                      (four 8-bit passes over order-preserving integer keys), then a stable
//                      compaction in token order -> chosen[e][0..C) ascending; per-token counts of
//                      the experts that chose it; the last block to finish writes dropped[t]
//   ec_gather_kernel   x rows into x_perm (row e*C + j = j-th token of expert e), row maps,
//                      offsets e*C, and clearing of out where the forward's GEMM1 does not zero it
//   ec_combine_kernel  unfused combine, token-major: out[t] = sum over the experts that chose t, in
//                      ascending order, of p[t,e] * y[row] (no atomics; the same bits on every run)
//
// The expert FFN that runs between gather and combine is the token-choice one: row_slot holds the
// expert and the combine weight of row r is topk_w[t * E + e] = p[t,e].
#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kSelThreads = 1024;  // the block scans below assume exactly 32 warps

// fp32 -> uint32 with the same order (larger float, larger key); -0 sorts just below +0
__device__ __forceinline__ uint32_t order_key(float v) {
  const uint32_t u = __float_as_uint(v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive count of `flag` over the block's threads in thread order; the block total goes to
// `total`.  `buf` holds at least 65 ints of shared memory.
__device__ __forceinline__ int block_excl_count(bool flag, int* buf, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned bal = __ballot_sync(0xffffffffu, flag);
  if (lane == 0) buf[warp] = __popc(bal);
  __syncthreads();
  if (warp == 0) {
    const int v = buf[lane];
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += n;
    }
    buf[32 + lane] = incl - v;
    if (lane == 31) buf[64] = incl;
  }
  __syncthreads();
  const int r = buf[32 + warp] + __popc(bal & ((1u << lane) - 1u));
  total = buf[64];
  __syncthreads();  // buf is reused by the next call
  return r;
}

__global__ void __launch_bounds__(kSelThreads) ec_select_kernel(EcSelectArgs a) {
  __shared__ int hist[256];
  __shared__ int buf[72];
  __shared__ uint32_t sel_digit;
  __shared__ int sel_need;
  __shared__ int is_last;
  const int e = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int T = a.T, C = a.C;
  const float* sc = a.scores + (size_t)e * T;
  const bool all = C >= T;

  // Radix select, most significant digit first.  Invariant: at least `need` of the tokens whose key
  // matches `prefix` under `mask` remain, and exactly C - need tokens have a larger key.
  uint32_t prefix = 0, mask = 0;
  int need = C;
  if (!all) {
    for (int pass = 0; pass < 4; ++pass) {
      const int shift = 24 - 8 * pass;
      for (int i = tid; i < 256; i += kSelThreads) hist[i] = 0;
      __syncthreads();
      for (int t = tid; t < T; t += kSelThreads) {
        const uint32_t key = order_key(sc[t]);
        if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1);
      }
      __syncthreads();
      if (warp == 0) {
        // lane l holds digits 255-8l .. 248-8l (largest first); the first lane whose running
        // count from the top reaches `need` holds the digit of the C-th largest key
        int cnt[8], sum = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          cnt[j] = hist[255 - 8 * lane - j];
          sum += cnt[j];
        }
        int incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int n = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += n;
        }
        const unsigned hit = __ballot_sync(0xffffffffu, incl >= need);
        if (lane == __ffs(hit) - 1) {
          int run = incl - sum;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            if (run + cnt[j] >= need) {
              sel_digit = (uint32_t)(255 - 8 * lane - j);
              sel_need = need - run;
              break;
            }
            run += cnt[j];
          }
        }
      }
      __syncthreads();
      prefix |= sel_digit << shift;
      mask |= 255u << shift;
      need = sel_need;
      __syncthreads();  // hist and sel_* are rewritten by the next pass
    }
  }
  const uint32_t thr = prefix;  // the C-th largest key; `need` tokens equal to it are taken

  // Stable compaction in token order: every key above thr, and the first `need` keys equal to it.
  int base_eq = 0, base_sel = 0;
  for (int t0 = 0; t0 < T; t0 += kSelThreads) {
    const int t = t0 + tid;
    const uint32_t key = t < T ? order_key(sc[t]) : 0u;
    const bool gt = t < T && (all || key > thr);
    const bool eq = t < T && !all && key == thr;
    int tot_eq, tot_sel;
    const int r_eq = base_eq + block_excl_count(eq, buf, tot_eq);
    const bool take = gt || (eq && r_eq < need);
    const int pos = base_sel + block_excl_count(take, buf, tot_sel);
    if (take) {
      a.chosen[(size_t)e * C + pos] = t;
      atomicAdd(&a.tok_count[t], 1);
    }
    base_eq += tot_eq;
    base_sel += tot_sel;
  }
  if (tid == 0) {
    a.expert_counts[e] = C;
    a.cnt_pre[e] = C;
  }

  // The last block to finish sees every expert's counts and writes the per-token flags.
  __threadfence();
  __syncthreads();
  if (tid == 0) is_last = atomicAdd(a.done, 1u) == gridDim.x - 1;
  __syncthreads();
  if (is_last) {
    __threadfence();
    for (int t = tid; t < T; t += kSelThreads) a.dropped[t] = __ldcg(&a.tok_count[t]) == 0 ? 1 : 0;
    if (tid == 0) *a.done = 0u;  // ready for the next call on this workspace
  }
}

// 32 rows per 256-thread block: row maps, 16-byte copies of the x rows into x_perm (8 loads in
// flight per thread), and a grid-stride clear of out.
__global__ void __launch_bounds__(256) ec_gather_kernel(EcGatherArgs a) {
  __shared__ int tok_s[32];
  const int tid = threadIdx.x;
  const long long rows = (long long)a.E * a.C;
  const long long r0 = (long long)blockIdx.x * 32;
  // block (x, z) copies columns slice z of rows 32x..32x+31; slice 0 writes the row maps
  const bool maps = blockIdx.y == 0;
  if (tid < 32) {
    const long long r = r0 + tid;
    int t = -1;
    if (r < rows) {
      t = a.chosen[r];
      if (t < 0 || t >= a.T) {  // caller-supplied token outside [0, T): a zero row for token 0, error recorded
        if (maps) atomicCAS(a.status, 0, kDevBadIndex);
        t = -1;
      }
      if (maps) {
        a.row_token[r] = t < 0 ? 0 : t;
        a.row_slot[r] = (int)(r / a.C);
      }
    }
    tok_s[tid] = t;
  }
  if (blockIdx.x == 0 && maps)
    for (int e = tid; e <= a.E; e += 256) a.offsets[e] = e * a.C;
  __syncthreads();
  if (a.out != nullptr) {
    // this block's share of out, interleaved over the grid; the stores go out before the copies
    const long long ovec = (long long)a.T * a.H / 4;
    const long long nb = (long long)gridDim.x * gridDim.y;
    const long long b = (long long)blockIdx.y * gridDim.x + blockIdx.x;
    float4* o = reinterpret_cast<float4*>(a.out);
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
    for (long long i = b * 256 + tid; i < ovec; i += nb * 256) o[i] = z;
  }
  const int nvec = a.H * a.esize / 16;
  const int c_lo = (int)((long long)nvec * blockIdx.y / gridDim.y);
  const int w = (int)((long long)nvec * (blockIdx.y + 1) / gridDim.y) - c_lo;
  const uint4* xv = reinterpret_cast<const uint4*>(a.x);
  uint4* pv = reinterpret_cast<uint4*>(a.x_perm);
  const int total = 32 * w;
  constexpr int U = 8;
  for (int i = tid; i < total; i += 256 * U) {
    uint4 v[U];
    int ok[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int idx = i + u * 256;
      ok[u] = 0;
      if (idx < total) {
        const int r = idx / w, c = c_lo + idx % w;
        if (tok_s[r] >= 0) {
          v[u] = xv[(size_t)tok_s[r] * nvec + c];
          ok[u] = 1;
        }
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int idx = i + u * 256;
      if (idx >= total) continue;
      const int r = idx / w, c = c_lo + idx % w;
      if (ok[u]) pv[(size_t)(r0 + r) * nvec + c] = v[u];
      else if (r0 + r < rows) pv[(size_t)(r0 + r) * nvec + c] = make_uint4(0u, 0u, 0u, 0u);  // invalid token
    }
  }
}

// One block per row: out[t] += p[t,e] * y[row] (fp32 atomics; up to E rows meet in a token).
// Token-major combine without atomics: block t finds, for every expert e, the row holding token t
// (binary search of the expert's ascending chosen list; -1 when e did not choose t), then writes
// out[t] = sum over those experts, in ascending order, of p[t,e] * y[row] -- one fixed order, so the
// result repeats bit for bit, and every out row is written exactly once (0 for a token no expert chose).
__global__ void __launch_bounds__(256) ec_combine_kernel(const float* __restrict__ y, const int32_t* __restrict__ chosen,
                                                         const float* __restrict__ topk_w, int E, int C, int H,
                                                         float* __restrict__ out) {
  __shared__ int rows_s[256];
  __shared__ float w_s[256];
  const int t = blockIdx.x;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int32_t* ch = chosen + (size_t)e * C;
    int lo = 0, hi = C;  // first position with ch[pos] >= t
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (ch[mid] < t) lo = mid + 1;
      else hi = mid;
    }
    const bool hit = lo < C && ch[lo] == t;
    rows_s[e] = hit ? e * C + lo : -1;
    w_s[e] = hit ? topk_w[(size_t)t * E + e] : 0.f;
  }
  __syncthreads();
  const int nv = H / 4;
  const float4* yv = reinterpret_cast<const float4*>(y);
  float4* ov = reinterpret_cast<float4*>(out) + (size_t)t * nv;
  for (int c = threadIdx.x; c < nv; c += blockDim.x) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int e = 0; e < E; ++e) {
      const int r = rows_s[e];
      if (r < 0) continue;
      const float w = w_s[e];
      const float4 v = yv[(size_t)r * nv + c];
      acc.x = fmaf(w, v.x, acc.x);
      acc.y = fmaf(w, v.y, acc.y);
      acc.z = fmaf(w, v.z, acc.z);
      acc.w = fmaf(w, v.w, acc.w);
    }
    ov[c] = acc;
  }
}

}  // namespace

cudaError_t launch_ec_select(const EcSelectArgs& a, cudaStream_t st) {
  ec_select_kernel<<<a.E, kSelThreads, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_ec_gather(const EcGatherArgs& a, cudaStream_t st) {
  const long long rows = (long long)a.E * a.C;
  // each 32-row block's columns split over up to 4 slices of at least 8 vectors (128 B): one or two
  // rounds of loads in flight per thread, as in the token-choice scatter
  const int nvec = a.H * a.esize / 16;
  int S = 1;
  while (S < 4 && nvec / (2 * S) >= 8) S *= 2;
  dim3 grid((unsigned)((rows + 31) / 32), (unsigned)S);
  ec_gather_kernel<<<grid, 256, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_ec_combine(const float* y, const int32_t* chosen, const float* topk_w, int T, int E, int C, int H,
                              float* out, cudaStream_t st) {
  if (T <= 0) return cudaSuccess;
  ec_combine_kernel<<<T, 256, 0, st>>>(y, chosen, topk_w, E, C, H, out);
  return cudaGetLastError();
}

}  // namespace moe

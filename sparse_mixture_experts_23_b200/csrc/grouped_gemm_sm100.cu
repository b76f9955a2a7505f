// Grouped expert GEMMs on the 5th-generation tensor cores (sm_100a: TMA + tcgen05.mma + TMEM).
//
// Expert FFN of the MoE layer ("MoE Training: Mixture of Experts" page, Quick Start expert
// Linear(H, 4H) -> GELU -> Linear(4H, H); Advanced Patterns Mixtral block: gather rows by expert,
// scale by the routing weight, index_add_ back to token order) over variable-length expert
// segments of the permuted rows:
//   GEMM1 (EPI_GELU):     h[r, n]   = bf16( GELU( sum_k x_perm[r,k] W1[e,k,n] + b1[e,n] ) )
//   GEMM1 (EPI_SILU):     the same with SiLU (Mixtral block experts); b1 and b2 may be absent (zero)
//   GEMM2 (EPI_COMBINE):  out[t, n] += w(t,s) * ( sum_k h[r,k] W2[e,k,n] + b2[e,n] ),  t,s = row r's
//   GEMM2 (EPI_STORE_Y):  y[r, n]   = sum_k h[r,k] W2[e,k,n] + b2[e,n]
//
// Design (one persistent CTA per SM, 64 + 32 * kEpiWarps threads: 192 with the default 4 epilogue warps):
//   warp 0      TMA producer: A tile [128 rows x 64 k] (K-major, 128B swizzle) and B tile
//               [64 k x BN n] (weights are stored n-contiguous, i.e. MN-major, 128B swizzle, loaded
//               as BN/64 boxes of 64x64) into a kStages-deep shared-memory ring.
//   warp 1      allocates 2*BN TMEM columns (two fp32 accumulators), one elected lane issues
//               tcgen05.mma kind::f16 (M=128, N=BN, K=16, bf16 x bf16 -> fp32) and tcgen05.commit
//               to release smem stages and to hand a finished accumulator to the epilogue.
//   warps 2..   epilogue (kEpiWarps = 4: warps 2..5, one per TMEM lane quarter; 8: two warps share
//               each quarter and split the tile's columns): tcgen05.ld 32 lanes x 32 columns per step
//               (each thread owns one row),
//               fused bias + GELU -> bf16 store, or bias + gate-weight scale + vector fp32 red.add
//               into out (at most k adds per element, so k <= 2 is order independent).
// Tiles run expert-major, then n-tile, then m-tile, so the CTAs in flight share one expert's
// weight columns and activation rows through L2.  Rows past an expert's segment inside its last
// m-tile are computed on whatever the buffer holds there and masked in the epilogue.
// Every mbarrier wait is bounded: a wait that runs out sets the workspace error word, raises a
// CTA-wide abort flag, and the CTA drains its in-flight copies / MMAs (bounded) and exits.
// Every TMA load brings one CTA its own tile; no load is shared across the CTAs of a cluster.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>
#include <math.h>
#include <stdlib.h>

#include "moe_internal.cuh"
#include "sm100_ptx.cuh"

namespace moe {

namespace {

constexpr int BM = 128;
constexpr int BK = 64;  // one 128-byte swizzle row of bf16
#ifndef MOE_EPI_WARPS
#define MOE_EPI_WARPS 4
#endif
constexpr int kEpiWarps = MOE_EPI_WARPS;  // 4 or 8: one or two warps per TMEM lane quarter
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int kStgStride = 36;                     // floats per staged row (32 + 4: 16-byte rows, spread banks)
constexpr int kStgWarpBytes = 5 * 1024;  // one warp's staging tile: 32 x 32 fp32 (padded rows) or a
                                          // 1024-aligned 32 x 64 bf16 box in 128-byte swizzle

enum {
  EPI_GELU = 0,
  EPI_COMBINE = 1,
  EPI_STORE_Y = 2,
  EPI_SILU = 3,
  EPI_DGRAD_GELU = 4,
  EPI_DGRAD_SILU = 5,
  EPI_ROUTER = 6  // the gate: softmax, top-k, renormalised weights and a chunk's loss partials
};
// GEMM1 epilogues write h = act(acc + b1); GEMM2 epilogues combine or store y; the backward's
// first GEMM (G = dout_rows . W2[e]^T) writes du = w * G * act'(u) and accumulates dw = G . h.
__host__ __device__ constexpr bool epi_h(int epi) { return epi == EPI_GELU || epi == EPI_SILU; }
__host__ __device__ constexpr bool epi_dgrad(int epi) { return epi == EPI_DGRAD_GELU || epi == EPI_DGRAD_SILU; }

template <int BN>
struct Cfg {
  static constexpr int kStages = BN == 256 ? 4 : (BN == 128 ? 6 : 8);  // as deep as shared memory allows
  static constexpr int kABytes = BM * BK * 2;
  static constexpr int kBBytes = BK * BN * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kTmemCols = 2 * BN;
  // smem: [align pad][A stages][B stages][barriers][tmem slot, abort][offsets, tile prefix]
  static constexpr int kBarOff = kStages * kStageBytes;
  static constexpr int kNumBars = 2 * kStages + 4 + 1;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kOffsOff = kMiscOff + 16;
  static constexpr int kStgOff = (kOffsOff + 2 * 260 * 4 + 127) & ~127;  // per-warp epilogue staging tiles
  static constexpr int kSmemBytes = 1024 + kStgOff + kEpiWarps * kStgWarpBytes;
  static_assert(kStgOff % 16 == 0 && kSmemBytes <= 232448, "shared-memory plan");
  // instruction descriptor, kind::f16: D fp32, A bf16 K-major, B bf16 MN-major, M=128, N=BN
  static constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (0u << 15) | (1u << 16) |
                                     ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
};

struct GemmArgs {
  const int32_t* offsets;
  int E, N, K;
  const __nv_bfloat16* bias;
  __nv_bfloat16* h_out;           // GEMM1: h; backward GEMM: du
  __nv_bfloat16* u_out;           // GEMM1 of a training forward: the pre-activation u (else null)
  const __nv_bfloat16* h_in;      // backward GEMM: the forward's h and u
  const __nv_bfloat16* u_in;
  float* dwraw;                   // backward GEMM: per-row sum_n G * h (atomically accumulated)
  float* out;
  float* y;
  const int32_t* row_token;
  const int32_t* row_slot;
  const float* topk_w;
  int k;
  int single_rows;  // offsets == null: one segment of this many rows (a plain dense GEMM)
  // EPI_ROUTER outputs (N = E experts in one tile; each epilogue warp's 32 rows are one 32-token chunk)
  int32_t* r_topk_idx;    // [T,k]
  float* r_topk_w;        // [T,k]
  float* r_loss_part;     // [nchunk][E+1]: sum_t p[t,e], then sum_t lse_t^2
  int32_t* r_chunk_hist;  // [k][nchunk][E]
  float* r_logits;        // [T,E] logits (training forward), or null
  int a_box_rows;   // single-CTA kernel: > 0 loads only ceil(rows / a_box_rows) boxes of that many A rows
  // single-CTA kernel, GEMM2 with the fused combine of a top-1 layer: > 1 splits every tile's K range
  // into that many parts, each its own work item adding its partial product into out (the bias with
  // part 0).  With k = 1 an element of out then receives exactly 2 adds, whose order does not matter.
  int k_splits;
  // single-CTA kernel, with a_box_rows = 8: segment rows 8j .. 8j+7 of a tile go to tile rows
  // 32*(j%4) + 8*(j/4) .., so the rows of a short segment spread over all four TMEM lane quarters and
  // every epilogue warp gets a share of them (else a 64-row segment leaves two of the four idle)
  int spread_rows;
  int32_t* status;
  long long wait_limit;
  // GEMM1 on CTA pairs: the epilogue warps zero clear[0, clear_n) before their first tile, while the
  // MMA warp runs that tile's main loop (the forward's out, which GEMM2 then accumulates into)
  float4* clear;
  long long clear_n;
};

using namespace sm100;

// Zeroes p[0, n) in 16-byte stores, the CTAs' 2 KB runs interleaved across the grid.
__device__ __noinline__ void clear_f4(float4* p, long long n, int cta, int ncta, int t) {
  const long long stride = (long long)ncta * (32 * kEpiWarps);
  const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
  for (long long i = (long long)cta * (32 * kEpiWarps) + t; i < n; i += stride) p[i] = z;
}

// Phi(u) = P(Z <= u) for a standard normal Z, so that GELU(u) = u Phi(u) = 0.5 u (1 + erf(u / sqrt 2)).
// erfc(x) for x >= 0 from Abramowitz & Stegun, Handbook of Mathematical Functions, 7.1.26 (Hastings):
//   erfc(x) = (a1 t + a2 t^2 + a3 t^3 + a4 t^4 + a5 t^5) exp(-x^2) + e(x),  t = 1 / (1 + p x),  |e(x)| <= 1.5e-7,
// at x = |u| / sqrt 2; Phi = 1 - erfc/2 for u >= 0 and erfc/2 below.  Two special-function-unit
// operations (reciprocal, exponential) and five FMAs: the GEMM1 epilogue evaluates this for every
// element of h, and on short-K tiles (the Switch shape) the epilogue sets the pace.
__device__ __forceinline__ float normal_cdf(float u) {
  const float x = fabsf(u) * 0.70710678118654752f;
  const float t = __fdividef(1.f, fmaf(0.3275911f, x, 1.f));
  float poly = fmaf(t, 1.061405429f, -1.453152027f);
  poly = fmaf(t, poly, 1.421413741f);
  poly = fmaf(t, poly, -0.284496736f);
  poly = fmaf(t, poly, 0.254829592f);
  const float half_erfc = 0.5f * poly * t * __expf(-x * x);
  return u >= 0.f ? 1.f - half_erfc : half_erfc;
}
__device__ __forceinline__ float gelu_erf(float u) { return u * normal_cdf(u); }
// u * sigmoid(u); for u < -87 the fast divide returns 0 where the exact value is below 1e-35
__device__ __forceinline__ float silu(float u) { return __fdividef(u, 1.f + __expf(-u)); }
template <int EPI>
__device__ __forceinline__ float act(float u) {
  if constexpr (EPI == EPI_SILU) return silu(u);
  else return gelu_erf(u);
}
// derivatives: GELU'(u) = Phi(u) + u phi(u); SiLU'(u) = s (1 + u (1 - s)), s = sigmoid(u)
__device__ __forceinline__ float gelu_grad(float u) {
  return normal_cdf(u) + u * 0.3989422804014327f * __expf(-0.5f * u * u);
}
__device__ __forceinline__ float silu_grad(float u) {
  const float sg = __fdividef(1.f, 1.f + __expf(-u));
  return sg * (1.f + u * (1.f - sg));
}
template <int EPI>
__device__ __forceinline__ float act_grad(float u) {
  if constexpr (EPI == EPI_DGRAD_SILU) return silu_grad(u);
  else return gelu_grad(u);
}
// 8 bias values at brow[n0 .. n0+8) as 4 bf16 pairs, zeros when the layer has no bias
__device__ __forceinline__ uint4 bias8(const __nv_bfloat16* brow, int n0) {
  return brow ? __ldg(reinterpret_cast<const uint4*>(brow + n0)) : make_uint4(0u, 0u, 0u, 0u);
}

// tile -> (expert, m tile inside the expert, n tile); prefix[e] = tiles of experts < e
__device__ __forceinline__ void decode_tile(int tile, const int* prefix, const int* offs, int E, int NT, int& e,
                                            int& m_local, int& n_idx, int& row0, int& rows) {
  int lo = 0, hi = E;  // find the last e with prefix[e] <= tile (skips empty experts)
  while (hi - lo > 1) {
    int mid = (lo + hi) >> 1;
    if (prefix[mid] <= tile) lo = mid;
    else hi = mid;
  }
  e = lo;
  const int cnt = offs[e + 1] - offs[e];
  const int mt = (cnt + BM - 1) / BM;
  const int local = tile - prefix[e];
  n_idx = local / mt;
  m_local = local % mt;
  row0 = offs[e] + m_local * BM;
  rows = min(BM, cnt - m_local * BM);
}

// Epilogue of one 32 x 32 accumulator chunk of a warp (lane i holds row i of the chunk in r[]).
// The chunk goes through the warp's shared staging tile so that, after the transpose, lane j owns
// column j and every global store or reduction writes one contiguous row segment:
//   EPI_GELU:    h[grow_i, n0 + j]   = bf16(GELU(acc + b1[n0 + j]))       (64 B per row; SiLU alike)
//   EPI_COMBINE: out[tok_i, n0 + j] += w_i * (acc + b2[n0 + j])           (128 B per row, fp32 red)
//   EPI_STORE_Y: y[grow_i, n0 + j]   = acc + b2[n0 + j]                   (128 B per row)
// Lane i's row is grow_i = grow0 + off_i with off_i = i, or with SPREAD (rows spread over the lane
// quarters in groups of 8) off_i = 32*(i/8) + i%8; rows with off_i >= nrows (past the expert's
// segment) are skipped.
template <int EPI, bool SPREAD = false>
__device__ __forceinline__ void epilogue_chunk(const GemmArgs& g, const uint32_t (&r)[32], float* stg, int lane,
                                               int grow0, int nrows, int my_tok, float my_w, const __nv_bfloat16* brow,
                                               int n0) {
  float4* mine = reinterpret_cast<float4*>(stg + lane * kStgStride);
#pragma unroll
  for (int q = 0; q < 8; ++q)
    mine[q] = make_float4(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]), __uint_as_float(r[4 * q + 2]),
                          __uint_as_float(r[4 * q + 3]));
  __syncwarp();
  const float bj = brow ? __bfloat162float(brow[n0 + lane]) : 0.f;
  const int nr = nrows < 32 ? nrows : 32;
  // 8 rows at a time: their values (and activations) are independent, so the latency of one row's
  // chain overlaps the others' (one warp per SM sub-partition runs this loop)
#pragma unroll 1
  for (int i0 = 0; i0 < 32; i0 += 8) {
    const int off0 = SPREAD ? 4 * i0 : i0;  // offset of row i0: 32 * (i0 / 8) with SPREAD
    if (off0 >= (SPREAD ? nrows : nr)) break;  // warp-uniform; later groups lie further out
    float v[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) v[q] = stg[(i0 + q) * kStgStride + lane] + bj;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int i = i0 + q, off = off0 + q;
      const bool ok = SPREAD ? off < nrows : i < nr;
      if constexpr (epi_h(EPI)) {
        const __nv_bfloat16 hv = __float2bfloat16_rn(act<EPI>(v[q]));
        if (ok) {
          g.h_out[(size_t)(grow0 + off) * g.N + n0 + lane] = hv;
          if (g.u_out) g.u_out[(size_t)(grow0 + off) * g.N + n0 + lane] = __float2bfloat16_rn(v[q]);
        }
      } else if (EPI == EPI_COMBINE) {
        const int tok = __shfl_sync(0xffffffffu, my_tok, i);
        const float w = __shfl_sync(0xffffffffu, my_w, i);
        if (ok) atomicAdd(g.out + (size_t)tok * g.N + n0 + lane, w * v[q]);
      } else {
        if (ok) g.y[(size_t)(grow0 + off) * g.N + n0 + lane] = v[q];
      }
    }
  }
  __syncwarp();
}

// GEMM1 epilogue of a 64-column group of a warp's 32 rows (lane i owns row i): bias + activation, bf16,
// written into the warp's staging box in the 128-byte swizzle a TMA store expects (16-byte piece
// j of row i sits at piece j ^ (i % 8)), then stored with one TMA instruction.  Only used when all
// 32 rows lie inside the expert's segment, so the box never touches the next expert's rows.
template <int EPI>
__device__ __forceinline__ void epilogue_h_box(const CUtensorMap* tmC, const uint32_t (&r0)[32],
                                                  const uint32_t (&r1)[32], uint8_t* stg, int lane,
                                                  const __nv_bfloat16* brow, int n0, int grow0,
                                                  __nv_bfloat16* u_out, int ldu) {
  if (lane == 0) bulk_wait_read0();  // the previous box has left the staging buffer
  __syncwarp();
  uint8_t* row = stg + lane * 128;
  uint4* urow = u_out ? reinterpret_cast<uint4*>(u_out + (size_t)(grow0 + lane) * ldu + n0) : nullptr;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint32_t* src = j < 4 ? &r0[8 * j] : &r1[8 * (j - 4)];
    const uint4 bb = bias8(brow, n0 + 8 * j);
    const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&bb);
    uint32_t w[4], uw[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float2 f = __bfloat1622float2(b2[u]);
      const float v0 = __uint_as_float(src[2 * u]) + f.x, v1 = __uint_as_float(src[2 * u + 1]) + f.y;
      const __nv_bfloat162 v = __floats2bfloat162_rn(act<EPI>(v0), act<EPI>(v1));
      w[u] = *reinterpret_cast<const uint32_t*>(&v);
      const __nv_bfloat162 pre = __floats2bfloat162_rn(v0, v1);
      uw[u] = *reinterpret_cast<const uint32_t*>(&pre);
    }
    *reinterpret_cast<uint4*>(row + ((j ^ (lane & 7)) * 16)) = make_uint4(w[0], w[1], w[2], w[3]);
    if (urow) urow[j] = make_uint4(uw[0], uw[1], uw[2], uw[3]);
  }
  fence_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(tmC, smem_u32(stg), n0, grow0);
    bulk_commit();
  }
}

// The same values written row by row from registers (rows past the segment are skipped).
template <int EPI>
__device__ __forceinline__ void epilogue_h_rows(const GemmArgs& g, const uint32_t (&r0)[32], const uint32_t (&r1)[32],
                                                   int lane, int nrows, const __nv_bfloat16* brow, int n0, int grow0) {
  if (lane >= nrows) return;
  uint4* dst = reinterpret_cast<uint4*>(g.h_out + (size_t)(grow0 + lane) * g.N + n0);
  uint4* urow = g.u_out ? reinterpret_cast<uint4*>(g.u_out + (size_t)(grow0 + lane) * g.N + n0) : nullptr;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint32_t* src = j < 4 ? &r0[8 * j] : &r1[8 * (j - 4)];
    const uint4 bb = bias8(brow, n0 + 8 * j);
    const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&bb);
    uint32_t w[4], uw[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float2 f = __bfloat1622float2(b2[u]);
      const float v0 = __uint_as_float(src[2 * u]) + f.x, v1 = __uint_as_float(src[2 * u + 1]) + f.y;
      const __nv_bfloat162 v = __floats2bfloat162_rn(act<EPI>(v0), act<EPI>(v1));
      w[u] = *reinterpret_cast<const uint32_t*>(&v);
      const __nv_bfloat162 pre = __floats2bfloat162_rn(v0, v1);
      uw[u] = *reinterpret_cast<const uint32_t*>(&pre);
    }
    dst[j] = make_uint4(w[0], w[1], w[2], w[3]);
    if (urow) urow[j] = make_uint4(uw[0], uw[1], uw[2], uw[3]);
  }
}

// Backward epilogue of 32 accumulator columns of one row (lane = row): G = acc is the row's
// dout . W2[e]^T at columns n0..n0+32; dw += G . h[row, cols]; du[row, cols] = bf16(w G act'(u)).
// h, u and du rows are read and written as 64-byte runs.
template <int EPI>
__device__ __forceinline__ void epilogue_dgrad32(const GemmArgs& g, const uint32_t (&r)[32], int grow, int n0, float w,
                                                 float& dw) {
  const uint4* hp = reinterpret_cast<const uint4*>(g.h_in + (size_t)grow * g.N + n0);
  const uint4* up = reinterpret_cast<const uint4*>(g.u_in + (size_t)grow * g.N + n0);
  uint4* dp = reinterpret_cast<uint4*>(g.h_out + (size_t)grow * g.N + n0);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint4 hv = __ldg(hp + j), uv = __ldg(up + j);
    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&hv);
    const __nv_bfloat162* u2 = reinterpret_cast<const __nv_bfloat162*>(&uv);
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 hf = __bfloat1622float2(h2[q]), uf = __bfloat1622float2(u2[q]);
      const float g0 = __uint_as_float(r[8 * j + 2 * q]), g1 = __uint_as_float(r[8 * j + 2 * q + 1]);
      dw = fmaf(g0, hf.x, fmaf(g1, hf.y, dw));
      const __nv_bfloat162 d = __floats2bfloat162_rn(w * g0 * act_grad<EPI>(uf.x), w * g1 * act_grad<EPI>(uf.y));
      o[q] = *reinterpret_cast<const uint32_t*>(&d);
    }
    dp[j] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// Gate tail of one epilogue warp: lane i owns token row_base + i, whose BN logits sit in TMEM
// columns [0, BN) of the warp's lane quarter.  The bias goes to the warp's staging area once (read
// back by broadcast); then three passes over TMEM: (1) the max and the top-k by (logit desc, index
// asc: a later expert displaces a candidate only when strictly larger), plus the logits themselves
// for a training forward; (2) e = exp(l - max) and their sum, the e written back over the
// accumulator; (3) p = e / sum, whose column sums over the warp's 32 tokens go through the staging
// tile (stored with a rotation so both the row writes and the column reads spread over the banks).
// Writes topk_idx / topk_w (renormalised over the k selected), the chunk's loss partials (sum_t
// p[t,e] for every expert, then sum_t lse^2) and its per-slot expert histograms -- the same
// quantities, in the same layout, as the CUDA-core router tail.
template <int BN>
__device__ __forceinline__ void router_epilogue(const GemmArgs& g, uint32_t taddr, float* stg, int lane, int row_base,
                                                int wrows) {
  constexpr int E = BN;
  const int k = g.k;
  const int t = row_base + lane;
  const bool ok = lane < wrows;
  const int chunk = row_base / 32;
  const int nchunk = (g.single_rows + 31) / 32;
  float* tile = stg;          // [32][32] fp32, rotated by row
  float* bias = stg + 1024;   // [E] fp32
  for (int e = lane; e < E; e += 32) bias[e] = g.bias ? __bfloat162float(g.bias[e]) : 0.f;
  __syncwarp();
  float cv[8];
  int ci[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    cv[i] = -INFINITY;
    ci[i] = 0x7fffffff;
  }
  float m = -INFINITY, kth = -INFINITY;
  // pass 1: max and the top-k candidates (experts visited in increasing order)
#pragma unroll 1
  for (int c = 0; c < BN / 32; ++c) {
    uint32_t r[32];
    tmem_ld32(taddr + c * 32, r);
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const int e = c * 32 + j;
      const float v = __uint_as_float(r[j]) + bias[e];
      r[j] = __float_as_uint(v);
      m = fmaxf(m, v);
      if (v > kth) {
        float nv = v;
        int ne = e;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          if (q < k && nv > cv[q]) {
            const float tv = cv[q];
            const int te = ci[q];
            cv[q] = nv;
            ci[q] = ne;
            nv = tv;
            ne = te;
          }
        }
#pragma unroll
        for (int q = 0; q < 8; ++q)
          if (q == k - 1) kth = cv[q];
      }
    }
    if (ok && g.r_logits) {
      float4* dst = reinterpret_cast<float4*>(g.r_logits + (size_t)t * E + c * 32);
#pragma unroll
      for (int q = 0; q < 8; ++q)
        dst[q] = make_float4(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]), __uint_as_float(r[4 * q + 2]),
                             __uint_as_float(r[4 * q + 3]));
    }
  }
  // pass 2: e = exp(l - max) written back over the accumulator, and their sum
  float ssum = 0.f;
#pragma unroll 1
  for (int c = 0; c < BN / 32; ++c) {
    uint32_t r[32];
    tmem_ld32(taddr + c * 32, r);
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const float ev = __expf(__uint_as_float(r[j]) + bias[c * 32 + j] - m);
      ssum += ev;
      r[j] = __float_as_uint(ev);
    }
    tmem_st32(taddr + c * 32, r);
  }
  const float inv_s = 1.f / ssum;
  const float lse = m + __logf(ssum);
  if (ok) {
    float psel = 0.f;
#pragma unroll
    for (int q = 0; q < 8; ++q)
      if (q < k) psel += __expf(cv[q] - m);
#pragma unroll
    for (int q = 0; q < 8; ++q)
      if (q < k) {
        g.r_topk_idx[(size_t)t * k + q] = ci[q];
        g.r_topk_w[(size_t)t * k + q] = __expf(cv[q] - m) / psel;
      }
  }
  // pass 3: p = e / sum -> per-expert sums over the chunk's tokens (column sums in a fixed order)
#pragma unroll 1
  for (int c = 0; c < BN / 32; ++c) {
    uint32_t r[32];
    tmem_ld32(taddr + c * 32, r);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float s4 = ok ? inv_s : 0.f;
      reinterpret_cast<float4*>(tile + lane * 32)[(q + lane) & 7] =
          make_float4(__uint_as_float(r[4 * q]) * s4, __uint_as_float(r[4 * q + 1]) * s4,
                      __uint_as_float(r[4 * q + 2]) * s4, __uint_as_float(r[4 * q + 3]) * s4);
    }
    __syncwarp();
    float col = 0.f;
    for (int i = 0; i < 32; ++i) col += tile[i * 32 + ((((lane >> 2) + i) & 7) << 2) + (lane & 3)];
    g.r_loss_part[(size_t)chunk * (E + 1) + c * 32 + lane] = col;
    __syncwarp();
  }
  float z = ok ? lse * lse : 0.f;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
  if (lane == 0) g.r_loss_part[(size_t)chunk * (E + 1) + E] = z;
  // per-slot expert histograms of the chunk: clear the rows, then one write per distinct expert
  for (int q = 0; q < k; ++q)
    for (int e = lane; e < E; e += 32) g.r_chunk_hist[((size_t)q * nchunk + chunk) * E + e] = 0;
  __syncwarp();
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    if (q < k) {
      const int key = ok ? ci[q] : -1 - lane;  // rows past the tokens never match
      const unsigned peers = __match_any_sync(0xffffffffu, key);
      if (ok && (__ffs(peers) - 1) == lane)
        g.r_chunk_hist[((size_t)q * nchunk + chunk) * E + ci[q]] = __popc(peers);
    }
  }
}


template <int BN, int EPI, bool BKM>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmA16, GemmArgs g) {
  using C = Cfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + C::kBarOff;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (C::kStages + s); };
  auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * C::kStages + b); };
  auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * C::kStages + 2 + b); };
  const uint32_t drain_bar = bar0 + 8u * (2 * C::kStages + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);
  int* offs = reinterpret_cast<int*>(smem + C::kOffsOff);
  int* prefix = offs + 260;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = g.E, NT = g.N / BN, KB = g.K / BK;
  float* stg = reinterpret_cast<float*>(smem + C::kStgOff + (warp >= 2 ? warp - 2 : 0) * kStgWarpBytes);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), kEpiWarps);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  for (int i = threadIdx.x; i <= E; i += kThreads) offs[i] = g.offsets ? g.offsets[i] : (i == 0 ? 0 : g.single_rows);
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
  __syncthreads();
  if (threadIdx.x == 0) {
    int run = 0;
    for (int e = 0; e < E; ++e) {
      prefix[e] = run;
      run += ((offs[e + 1] - offs[e] + BM - 1) / BM) * NT;
    }
    prefix[E] = run;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // work items: every tile, or every (tile, K part) with split K
  const int KS = g.k_splits > 1 ? g.k_splits : 1;
  const int total = prefix[E] * KS;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer -----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int armed[C::kStages];
      for (int s = 0; s < C::kStages; ++s) armed[s] = -1;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        int e, m_local, n_idx, row0, rows;
        decode_tile(tile / KS, prefix, offs, E, NT, e, m_local, n_idx, row0, rows);
        const int kb0 = KB * (tile % KS) / KS, kb1 = KB * (tile % KS + 1) / KS;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, g.wait_limit, abort_flag, g.status, kDevTimeoutProducer)) {
            ok = false;
            break;
          }
          const uint32_t a_dst = sbase + stage * C::kABytes;
          const uint32_t b_dst = sbase + C::kStages * C::kABytes + stage * C::kBBytes;
          armed[stage] = (int)phase;
          if (g.a_box_rows > 0) {
            // small segments: only the boxes that hold the tile's rows (the MMA's other A rows are
            // stale shared memory; their accumulator rows are never stored)
            const int nb = (rows + g.a_box_rows - 1) / g.a_box_rows;
            mbar_arrive_expect_tx(full_bar(stage), (uint32_t)(nb * g.a_box_rows * BK * 2 + C::kBBytes));
            for (int j = 0; j < nb; ++j) {
              // spread: 8-row group j at tile row 32*(j%4) + 8*(j/4) (a multiple of 8 rows, so the
              // 128-byte swizzle phase of every row is unchanged)
              const int trow = g.spread_rows ? 32 * (j & 3) + 8 * (j >> 2) : j * g.a_box_rows;
              tma_load_2d(a_dst + trow * 128, &tmA16, kb * BK, row0 + j * g.a_box_rows, full_bar(stage));
            }
          } else {
            mbar_arrive_expect_tx(full_bar(stage), C::kStageBytes);
            tma_load_2d(a_dst, &tmA, kb * BK, row0, full_bar(stage));
          }
          if constexpr (BKM) {
            // B stored [E][N][K]: one 64 k x BN rows box, k contiguous
            tma_load_3d(b_dst, &tmB, kb * BK, n_idx * BN, e, full_bar(stage));
          } else {
#pragma unroll
            for (int j = 0; j < BN / 64; ++j)
              tma_load_3d(b_dst + j * (BK * 128), &tmB, n_idx * BN + j * 64, kb * BK, e, full_bar(stage));
          }
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok || *abort_flag) {
        // drain: every armed stage's copies must land before the CTA exits
        for (int s = 0; s < C::kStages; ++s)
          if (armed[s] >= 0) {
            volatile int dummy = 0;
            mbar_wait(full_bar(s), (uint32_t)armed[s], g.wait_limit, &dummy, g.status, kDevTimeoutDrain);
          }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer -------------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      bool issued = false;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x, ++it) {
        const int buf = it & 1;
        const uint32_t tphase = (uint32_t)((it >> 1) & 1);
        if (!mbar_wait(tempty_bar(buf), tphase ^ 1u, g.wait_limit, abort_flag, g.status, kDevTimeoutMma)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(buf * BN);
        const int kb0 = KB * (tile % KS) / KS, kb1 = KB * (tile % KS + 1) / KS;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(full_bar(stage), phase, g.wait_limit, abort_flag, g.status, kDevTimeoutMma)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = sbase + stage * C::kABytes;
          const uint32_t b_addr = sbase + C::kStages * C::kABytes + stage * C::kBBytes;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t bdesc =
                BKM ? desc_a_kmajor(b_addr + kk * 32) : desc_mnmajor(b_addr + kk * 16 * 128, BK * 128);
            mma_bf16(d_tmem, desc_a_kmajor(a_addr + kk * 32), bdesc, BKM ? (C::kIdesc & ~(1u << 16)) : C::kIdesc,
                     (kb != kb0 || kk != 0) ? 1u : 0u);
          }
          issued = true;
          mma_commit(empty_bar(stage));
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit(tfull_bar(buf));
      }
      if ((!ok || *abort_flag) && issued) {
        // drain: MMAs still running must finish before TMEM is released
        mma_commit(drain_bar);
        volatile int dummy = 0;
        mbar_wait(drain_bar, 0, g.wait_limit, &dummy, g.status, kDevTimeoutDrain);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..5) --------
    const int quarter = warp & 3;  // TMEM lanes [32*quarter, 32*quarter + 32)
    const int half = (warp - 2) >> 2;  // which half of the tile's columns this warp handles
    const bool spread = g.spread_rows != 0;
    // the tile row (segment row inside the tile) whose accumulator sits in this lane
    const int r_in_tile = spread ? 8 * quarter + 32 * (lane >> 3) + (lane & 7) : quarter * 32 + lane;
    const int wbase = spread ? 8 * quarter : 32 * quarter;  // epilogue_chunk's grow0 offset for this warp
    int it = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++it) {
      int e, m_local, n_idx, row0, rows;
      decode_tile(tile / KS, prefix, offs, E, NT, e, m_local, n_idx, row0, rows);
      const int buf = it & 1;
      const uint32_t tphase = (uint32_t)((it >> 1) & 1);
      // every lane waits; the warp leaves together if any lane gave up (tcgen05.ld is warp-wide)
      const bool got = mbar_wait(tfull_bar(buf), tphase, g.wait_limit, abort_flag, g.status, kDevTimeoutEpilogue);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const bool row_ok = r_in_tile < rows;
      const int grow = row0 + r_in_tile;
      float wgt = 0.f;
      int tok = 0;
      if ((EPI == EPI_COMBINE || epi_dgrad(EPI)) && row_ok) {
        tok = g.row_token[grow];
        wgt = g.topk_w ? g.topk_w[(size_t)tok * g.k + g.row_slot[grow]] : 1.f;  // no weights: plain scatter-add
      }
      const __nv_bfloat16* brow = (g.bias && tile % KS == 0) ? g.bias + (size_t)e * g.N : nullptr;  // part 0 adds it
      const int wrows = rows - wbase;  // > 0: some of this warp's 32 rows lie inside the segment
      constexpr int kChunks = BN / 32 / (kEpiWarps / 4);  // 32-column chunks per epilogue warp
      float dw = 0.f;
      if constexpr (EPI == EPI_ROUTER) {
        // one 32-token chunk per warp (the tile's rows start at a multiple of 128); with 8 epilogue
        // warps the second warp of each lane quarter has nothing to do
        if (half == 0 && wrows > 0)
          router_epilogue<BN>(g, tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * BN), stg, lane,
                              row0 + quarter * 32, wrows);
      } else
#pragma unroll 1
      for (int c = half * kChunks; c < (half + 1) * kChunks; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * BN + c * 32), r);
        if constexpr (epi_dgrad(EPI)) {
          if (row_ok) epilogue_dgrad32<EPI>(g, r, grow, n_idx * BN + c * 32, wgt, dw);
        } else {
          if (wrows > 0) {
            if (spread)
              epilogue_chunk<EPI, true>(g, r, stg, lane, row0 + wbase, wrows, tok, wgt, brow, n_idx * BN + c * 32);
            else
              epilogue_chunk<EPI>(g, r, stg, lane, row0 + wbase, wrows, tok, wgt, brow, n_idx * BN + c * 32);
          }
        }
      }
      if constexpr (epi_dgrad(EPI)) {
        if (row_ok) atomicAdd(g.dwraw + grow, dw);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty_bar(buf));
    }
  }

  tc_fence_before();
  __syncthreads();
  __syncwarp();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// ------------------------------------------------------------------------------------------------
// CTA-pair variant: a cluster of 2 CTAs on one TPC computes a 256 x 256 tile with
// tcgen05.mma.cta_group::2 (M=256, N=256, K=16).  Each CTA loads its own 128 rows of A and its
// own 128 columns of B (so each SM streams half of B), and each CTA's TMEM receives the fp32
// accumulator of its 128 rows.  Shared-memory traffic per FLOP falls by a third against the
// single-CTA 128 x 256 tile, which is what lets the tensor pipe run near its rate.
//   leader (rank 0): arms the full barriers with both CTAs' bytes, issues the MMAs, commits to
//                    the empty / accumulator-full barriers of both CTAs;
//   both CTAs:       TMA producer (completion counted on the leader's full barrier), epilogue
//                    on their own rows (released to the leader's accumulator-empty barrier).
struct PairCfg {
  static constexpr int kTileM = 256, kTileN = 256;
  static constexpr int kHalfN = 128;  // B columns held by each CTA
  static constexpr int kSubK = 2;     // 64-wide K sub-blocks per pipeline stage
  static constexpr int kStageK = kSubK * BK;
#ifndef MOE_PAIR_STAGES
#define MOE_PAIR_STAGES 3
#endif
  static constexpr int kStages = MOE_PAIR_STAGES;
  static constexpr int kASubBytes = BM * BK * 2;       // 16 KB: 128 rows x 64 k
  static constexpr int kBSubBytes = BK * kHalfN * 2;   // 16 KB: 64 k x 128 columns (two 64x64 boxes)
  static constexpr int kABytes = kSubK * kASubBytes;   // 32 KB
  static constexpr int kBBytes = kSubK * kBSubBytes;   // 32 KB
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kTmemCols = 2 * kTileN;
  static constexpr int kBarOff = kStages * kStageBytes;
  static constexpr int kNumBars = 2 * kStages + 4 + 1;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kOffsOff = kMiscOff + 16;
  static constexpr int kStgOff = (kOffsOff + 2 * 260 * 4 + 1023) & ~1023;
  static constexpr int kSmemBytes = 1024 + kStgOff + kEpiWarps * kStgWarpBytes;
  static_assert(kStgOff % 1024 == 0 && kSmemBytes <= 232448, "shared-memory plan");
  static constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (0u << 15) | (1u << 16) |
                                     ((uint32_t)(kTileN >> 3) << 17) | ((uint32_t)(kTileM >> 4) << 24);
  // half tile (M = 128 over the pair, 64 rows per CTA) for an expert's last <= 128 rows
  static constexpr uint32_t kIdescHalf = (1u << 4) | (1u << 7) | (1u << 10) | (0u << 15) | (1u << 16) |
                                         ((uint32_t)(kTileN >> 3) << 17) | ((uint32_t)((kTileM / 2) >> 4) << 24);
};

__device__ __forceinline__ void decode_tile_m(int tile, const int* prefix, const int* offs, int E, int NT, int tile_m,
                                              int& e, int& m_local, int& n_idx, int& row0, int& rows) {
  int lo = 0, hi = E;
  while (hi - lo > 1) {
    int mid = (lo + hi) >> 1;
    if (prefix[mid] <= tile) lo = mid;
    else hi = mid;
  }
  e = lo;
  const int cnt = offs[e + 1] - offs[e];
  const int mt = (cnt + tile_m - 1) / tile_m;
  const int local = tile - prefix[e];
  n_idx = local / mt;
  m_local = local % mt;
  row0 = offs[e] + m_local * tile_m;
  rows = min(tile_m, cnt - m_local * tile_m);
}

template <int EPI, bool BKM>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                             const __grid_constant__ CUtensorMap tmC, GemmArgs g) {
  using C = PairCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + C::kBarOff;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (C::kStages + s); };
  auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * C::kStages + b); };
  auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * C::kStages + 2 + b); };
  const uint32_t drain_bar = bar0 + 8u * (2 * C::kStages + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);
  int* offs = reinterpret_cast<int*>(smem + C::kOffsOff);
  int* prefix = offs + 260;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* stg = reinterpret_cast<float*>(smem + C::kStgOff + (warp >= 2 ? warp - 2 : 0) * kStgWarpBytes);
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cluster_id = blockIdx.x >> 1, nclusters = gridDim.x >> 1;
  const int E = g.E, NT = g.N / C::kTileN, KB = g.K / C::kStageK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), 2 * kEpiWarps);  // every epilogue warp of both CTAs of the pair
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  for (int i = threadIdx.x; i <= E; i += kThreads) offs[i] = g.offsets[i];
  if (warp == 1) tmem_alloc_pair(smem_u32(tmem_slot), C::kTmemCols);
  __syncthreads();
  if (threadIdx.x == 0) {
    int run = 0;
    for (int e = 0; e < E; ++e) {
      prefix[e] = run;
      run += ((offs[e + 1] - offs[e] + C::kTileM - 1) / C::kTileM) * NT;
    }
    prefix[E] = run;
  }
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers are initialised before any cross-CTA signal
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = prefix[E];

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs) -----
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int armed[C::kStages];
      for (int s = 0; s < C::kStages; ++s) armed[s] = -1;
      bool ok = true;
      for (int tile = cluster_id; tile < total && ok; tile += nclusters) {
        int e, m_local, n_idx, row0, rows;
        decode_tile_m(tile, prefix, offs, E, NT, C::kTileM, e, m_local, n_idx, row0, rows);
        const int cta_rows = rows <= C::kTileM / 2 ? C::kTileM / 4 : C::kTileM / 2;  // rows per CTA: 64 or 128
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, g.wait_limit, abort_flag, g.status, kDevTimeoutProducer)) {
            ok = false;
            break;
          }
          const uint32_t a_dst = sbase + stage * C::kABytes;
          const uint32_t b_dst = sbase + C::kStages * C::kABytes + stage * C::kBBytes;
          if (leader) {
            mbar_arrive_expect_tx(full_bar(stage), 2 * C::kStageBytes);
            armed[stage] = (int)phase;
          }
          const uint32_t fb = peer_addr(full_bar(stage), 0);
#pragma unroll
          for (int sk = 0; sk < C::kSubK; ++sk) {
            const int k0 = kb * C::kStageK + sk * BK;
            tma_load_2d_pair(a_dst + sk * C::kASubBytes, &tmA, k0, row0 + cta_rows * (int)rank, fb);
            if constexpr (BKM) {
              // B stored [E][N][K]: this CTA's 128 columns as one 64 k x 128 rows box, k contiguous
              tma_load_3d_pair(b_dst + sk * C::kBSubBytes, &tmB, k0, n_idx * C::kTileN + C::kHalfN * (int)rank, e, fb);
            } else {
#pragma unroll
              for (int j = 0; j < C::kHalfN / 64; ++j)
                tma_load_3d_pair(b_dst + sk * C::kBSubBytes + j * (BK * 128), &tmB,
                                 n_idx * C::kTileN + C::kHalfN * (int)rank + j * 64, k0, e, fb);
            }
          }
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (leader && (!ok || *abort_flag)) {
        for (int s = 0; s < C::kStages; ++s)
          if (armed[s] >= 0) {
            volatile int dummy = 0;
            mbar_wait(full_bar(s), (uint32_t)armed[s], g.wait_limit, &dummy, g.status, kDevTimeoutDrain);
          }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader only) -----
    if (leader && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      bool issued = false;
      for (int tile = cluster_id; tile < total && ok; tile += nclusters, ++it) {
        const int buf = it & 1;
        const uint32_t tphase = (uint32_t)((it >> 1) & 1);
        int e_, m_l, n_i, r0_, rows;
        decode_tile_m(tile, prefix, offs, E, NT, C::kTileM, e_, m_l, n_i, r0_, rows);
        const uint32_t idesc0 = rows <= C::kTileM / 2 ? C::kIdescHalf : C::kIdesc;
        const uint32_t idesc = BKM ? (idesc0 & ~(1u << 16)) : idesc0;  // bit 16: B is MN-major
        if (!mbar_wait(tempty_bar(buf), tphase ^ 1u, g.wait_limit, abort_flag, g.status, kDevTimeoutMma)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(buf * C::kTileN);
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(full_bar(stage), phase, g.wait_limit, abort_flag, g.status, kDevTimeoutMma)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = sbase + stage * C::kABytes;
          const uint32_t b_addr = sbase + C::kStages * C::kABytes + stage * C::kBBytes;
#pragma unroll
          for (int kk = 0; kk < C::kStageK / 16; ++kk) {
            const int sk = kk / (BK / 16), ks = kk % (BK / 16);
            const uint64_t bdesc = BKM ? desc_a_kmajor(b_addr + sk * C::kBSubBytes + ks * 32)
                                       : desc_mnmajor(b_addr + sk * C::kBSubBytes + ks * 16 * 128, BK * 128);
            mma_bf16_pair(d_tmem, desc_a_kmajor(a_addr + sk * C::kASubBytes + ks * 32), bdesc, idesc,
                          (kb | kk) != 0 ? 1u : 0u);
          }
          issued = true;
          mma_commit_both(empty_bar(stage));  // frees this stage in both CTAs once its MMAs are done
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit_both(tfull_bar(buf));
      }
      if ((!ok || *abort_flag) && issued) {
        mma_commit_pair(drain_bar);
        volatile int dummy = 0;
        mbar_wait(drain_bar, 0, g.wait_limit, &dummy, g.status, kDevTimeoutDrain);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..5, both) --
    if constexpr (epi_h(EPI)) {
      if (g.clear != nullptr) clear_f4(g.clear, g.clear_n, (int)blockIdx.x, (int)gridDim.x, (int)threadIdx.x - 64);
    }
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;
    const uint32_t tempty_leader0 = peer_addr(tempty_bar(0), 0);
    const uint32_t tempty_leader1 = peer_addr(tempty_bar(1), 0);
    int it = 0;
    for (int tile = cluster_id; tile < total; tile += nclusters, ++it) {
      int e, m_local, n_idx, row0, rows;
      decode_tile_m(tile, prefix, offs, E, NT, C::kTileM, e, m_local, n_idx, row0, rows);
      const int buf = it & 1;
      const uint32_t tphase = (uint32_t)((it >> 1) & 1);
      const bool got = mbar_wait(tfull_bar(buf), tphase, g.wait_limit, abort_flag, g.status, kDevTimeoutEpilogue);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      // Full tile: this CTA's 128 rows in TMEM lanes 0..127, 256 columns.  Half tile (M = 128 over the
      // pair): this CTA's 64 rows x 256 columns sit in 128 TMEM columns, lanes 0..63 holding columns
      // 0..127 and lanes 64..127 columns 128..255 -- so lane quarter q has rows 32*(q%2).. and
      // columns 128*(q/2)..
      const bool hm = rows <= C::kTileM / 2;
      const int cta_rows = hm ? C::kTileM / 4 : C::kTileM / 2;
      const int qr = hm ? (quarter & 1) : quarter;  // 32-row block of this warp inside the CTA's rows
      const int colbase = hm ? (quarter >> 1) * (C::kTileN / 2) : 0;
      const int my_rows = min(rows - cta_rows * (int)rank, cta_rows);  // may be <= 0
      const int r_in = qr * 32 + lane;
      const bool row_ok = r_in < my_rows;
      const int grow = row0 + cta_rows * (int)rank + r_in;
      float wgt = 0.f;
      int tok = 0;
      if ((EPI == EPI_COMBINE || epi_dgrad(EPI)) && row_ok) {
        tok = g.row_token[grow];
        wgt = g.topk_w ? g.topk_w[(size_t)tok * g.k + g.row_slot[grow]] : 1.f;  // no weights: plain scatter-add
      }
      const __nv_bfloat16* brow = g.bias ? g.bias + (size_t)e * g.N : nullptr;
      const int wrows = my_rows - qr * 32;  // rows of this warp's 32 that lie inside the segment
      const int wrow0 = row0 + cta_rows * (int)rank + qr * 32;
      const int nch = (hm ? C::kTileN / 64 : C::kTileN / 32) / (kEpiWarps / 4);  // 32-column chunks per warp
      const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * C::kTileN);
      if constexpr (epi_h(EPI)) {
#pragma unroll 1
        for (int c = half * nch; c < (half + 1) * nch; c += 2) {
          uint32_t r0[32], r1[32];
          tmem_ld32(taddr + c * 32, r0);
          tmem_ld32(taddr + (c + 1) * 32, r1);
          const int n0 = n_idx * C::kTileN + colbase + c * 32;
          if (wrows >= 32)
            epilogue_h_box<EPI>(&tmC, r0, r1, reinterpret_cast<uint8_t*>(stg), lane, brow, n0, wrow0, g.u_out, g.N);
          else if (wrows > 0) epilogue_h_rows<EPI>(g, r0, r1, lane, wrows, brow, n0, wrow0);
        }
      } else if constexpr (epi_dgrad(EPI)) {
        float dw = 0.f;
#pragma unroll 1
        for (int c = half * nch; c < (half + 1) * nch; ++c) {
          uint32_t r[32];
          tmem_ld32(taddr + c * 32, r);
          if (row_ok) epilogue_dgrad32<EPI>(g, r, grow, n_idx * C::kTileN + colbase + c * 32, wgt, dw);
        }
        if (row_ok) atomicAdd(g.dwraw + grow, dw);
      } else {
#pragma unroll 1
        for (int c = half * nch; c < (half + 1) * nch; ++c) {
          uint32_t r[32];
          tmem_ld32(taddr + c * 32, r);
          if (wrows > 0)
            epilogue_chunk<EPI>(g, r, stg, lane, wrow0, wrows, tok, wgt, brow, n_idx * C::kTileN + colbase + c * 32);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(buf ? tempty_leader1 : tempty_leader0);
    }
    if (epi_h(EPI) && lane == 0) bulk_wait0();  // this warp's h boxes are written before exit
  }

  tc_fence_before();
  __syncthreads();
  __syncwarp();
  cluster_sync_all();  // neither CTA frees TMEM or exits while the pair still uses it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, C::kTmemCols);
  }
}

// ------------------------------------------------------------------ weight gradients ----------
// D[e] (M x N, fp32, row-major) = A_e^T . B_e for every expert, where A_e and B_e are the expert's
// rows offs[e]..offs[e+1] of A [rows, M] and B [rows, N] (both stored row-major, so both operands
// are MN-major).  The contraction runs over the expert's rows in 64-row blocks; rows of the last
// block past the segment belong to the next expert (or were never written), so the MMA warp zeroes
// them in shared memory after the TMA lands and before the MMAs read it.  Tiles are 128 x 256, m
// fastest inside an n column, expert-major; an expert with no rows gets zeros.  M and N are
// multiples of 64: partial tiles read zeros past the edge and the epilogue masks them.
struct WgCfg {
  static constexpr int kTileM = 128, kTileN = 256, kBK = 64;
  static constexpr int kStages = 4;
  static constexpr int kBoxBytes = 64 * kBK * 2;              // one 64 (m or n) x 64 (k) box: 8 KB
  static constexpr int kABytes = (kTileM / 64) * kBoxBytes;   // 16 KB
  static constexpr int kBBytes = (kTileN / 64) * kBoxBytes;   // 32 KB
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kTmemCols = 2 * kTileN;
  static constexpr int kBarOff = kStages * kStageBytes;
  static constexpr int kNumBars = 2 * kStages + 4 + 1;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kOffsOff = kMiscOff + 16;
  static constexpr int kStgOff = (kOffsOff + 260 * 4 + 127) & ~127;
  static constexpr int kSmemBytes = 1024 + kStgOff + kEpiWarps * kStgWarpBytes;
  static_assert(kStgOff % 16 == 0 && kSmemBytes <= 232448, "shared-memory plan");
  // kind::f16: D fp32, A and B bf16, both MN-major (bits 15, 16), N = 256, M = 128
  static constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) |
                                     ((uint32_t)(kTileN >> 3) << 17) | ((uint32_t)(kTileM >> 4) << 24);
};

struct WgradArgs {
  const int32_t* offsets;
  int E, M, N;
  float* out;  // [E][M][N]
  int32_t* status;
  long long wait_limit;
};

__global__ void __launch_bounds__(kThreads, 1)
    wgrad_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, WgradArgs g) {
  using C = WgCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + C::kBarOff;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (C::kStages + s); };
  auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * C::kStages + b); };
  auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * C::kStages + 2 + b); };
  const uint32_t drain_bar = bar0 + 8u * (2 * C::kStages + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);
  int* offs = reinterpret_cast<int*>(smem + C::kOffsOff);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* stg = reinterpret_cast<float*>(smem + C::kStgOff + (warp >= 2 ? warp - 2 : 0) * kStgWarpBytes);
  const int E = g.E;
  const int MT = (g.M + C::kTileM - 1) / C::kTileM, NT = (g.N + C::kTileN - 1) / C::kTileN;
  const int per_e = MT * NT;
  const int total = E * per_e;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), kEpiWarps);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  for (int i = threadIdx.x; i <= E; i += kThreads) offs[i] = g.offsets[i];
  if (warp == 1) tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  auto decode = [&](int tile, int& e, int& m0, int& n0) {
    e = tile / per_e;
    const int local = tile - e * per_e;
    n0 = (local / MT) * C::kTileN;
    m0 = (local % MT) * C::kTileM;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer -----------------
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int armed[C::kStages];
      for (int s = 0; s < C::kStages; ++s) armed[s] = -1;
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        int e, m0, n0;
        decode(tile, e, m0, n0);
        const int r0 = offs[e], KB = (offs[e + 1] - r0 + C::kBK - 1) / C::kBK;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, g.wait_limit, abort_flag, g.status, kDevTimeoutProducer)) {
            ok = false;
            break;
          }
          const uint32_t a_dst = sbase + stage * C::kStageBytes;
          const uint32_t b_dst = a_dst + C::kABytes;
          mbar_arrive_expect_tx(full_bar(stage), C::kStageBytes);
          armed[stage] = (int)phase;
          const int k0 = r0 + kb * C::kBK;
#pragma unroll
          for (int j = 0; j < C::kTileM / 64; ++j) tma_load_2d(a_dst + j * C::kBoxBytes, &tmA, m0 + j * 64, k0, full_bar(stage));
#pragma unroll
          for (int j = 0; j < C::kTileN / 64; ++j) tma_load_2d(b_dst + j * C::kBoxBytes, &tmB, n0 + j * 64, k0, full_bar(stage));
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok || *abort_flag) {
        for (int s = 0; s < C::kStages; ++s)
          if (armed[s] >= 0) {
            volatile int dummy = 0;
            mbar_wait(full_bar(s), (uint32_t)armed[s], g.wait_limit, &dummy, g.status, kDevTimeoutDrain);
          }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (whole warp) -------
    // All lanes wait on each stage; on a segment's last block they zero the rows past it, then
    // lane 0 issues the MMAs.
    int stage = 0;
    uint32_t phase = 0;
    int it = 0;
    bool ok = true;
    bool issued = false;
    for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x, ++it) {
      int e, m0, n0;
      decode(tile, e, m0, n0);
      const int r0 = offs[e], cnt = offs[e + 1] - r0, KB = (cnt + C::kBK - 1) / C::kBK;
      const int buf = it & 1;
      const uint32_t tphase = (uint32_t)((it >> 1) & 1);
      if (!__all_sync(0xffffffffu, mbar_wait(tempty_bar(buf), tphase ^ 1u, g.wait_limit, abort_flag, g.status,
                                             kDevTimeoutMma))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + (uint32_t)(buf * C::kTileN);
      for (int kb = 0; kb < KB; ++kb) {
        if (!__all_sync(0xffffffffu, mbar_wait(full_bar(stage), phase, g.wait_limit, abort_flag, g.status,
                                               kDevTimeoutMma))) {
          ok = false;
          break;
        }
        const uint32_t a_addr = sbase + stage * C::kStageBytes;
        const uint32_t b_addr = a_addr + C::kABytes;
        const int valid = min(C::kBK, cnt - kb * C::kBK);
        if (valid < C::kBK) {
          // rows valid..63 of every box: whole 128-byte lines (the swizzle permutes within a line)
          const int per_box = (C::kBK - valid) * 8;  // 16-byte pieces per box
          const int nbox = (C::kTileM + C::kTileN) / 64;
          for (int i = lane; i < nbox * per_box; i += 32) {
            const int box = i / per_box, rem = i - box * per_box;
            const uint32_t addr = a_addr + box * C::kBoxBytes + (valid + rem / 8) * 128 + (rem % 8) * 16;
            asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};\n" ::"r"(addr), "r"(0u) : "memory");
          }
          fence_async_smem();
        }
        __syncwarp();
        tc_fence_after();
        if (lane == 0) {
#pragma unroll
          for (int kk = 0; kk < C::kBK / 16; ++kk)
            mma_bf16(d_tmem, desc_mnmajor(a_addr + kk * 16 * 128, C::kBoxBytes),
                     desc_mnmajor(b_addr + kk * 16 * 128, C::kBoxBytes), C::kIdesc, (kb | kk) != 0 ? 1u : 0u);
          mma_commit(empty_bar(stage));
        }
        issued = true;
        __syncwarp();
        if (++stage == C::kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      if (lane == 0) mma_commit(tfull_bar(buf));  // with no rows this arrives at once; the epilogue writes zeros
      __syncwarp();
    }
    if ((!ok || *abort_flag) && issued && lane == 0) {
      mma_commit(drain_bar);
      volatile int dummy = 0;
      mbar_wait(drain_bar, 0, g.wait_limit, &dummy, g.status, kDevTimeoutDrain);
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..5) --------
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;
    int it = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++it) {
      int e, m0, n0;
      decode(tile, e, m0, n0);
      const bool empty = offs[e + 1] == offs[e];
      const int buf = it & 1;
      const uint32_t tphase = (uint32_t)((it >> 1) & 1);
      const bool got = mbar_wait(tfull_bar(buf), tphase, g.wait_limit, abort_flag, g.status, kDevTimeoutEpilogue);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const int row0 = m0 + quarter * 32;  // this warp's 32 rows of D
      const int nrows = min(32, g.M - row0);
      float* dst = g.out + (size_t)e * g.M * g.N;
      constexpr int kChunks = C::kTileN / 32 / (kEpiWarps / 4);
#pragma unroll 1
      for (int c = half * kChunks; c < (half + 1) * kChunks; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * C::kTileN + c * 32), r);
        const int col = n0 + c * 32;
        if (nrows <= 0 || col >= g.N) continue;
        // transpose through the warp's staging tile so that each store covers 128 contiguous bytes
        float4* mine = reinterpret_cast<float4*>(stg + lane * kStgStride);
#pragma unroll
        for (int q = 0; q < 8; ++q)
          mine[q] = empty ? make_float4(0.f, 0.f, 0.f, 0.f)
                          : make_float4(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]),
                                        __uint_as_float(r[4 * q + 2]), __uint_as_float(r[4 * q + 3]));
        __syncwarp();
        for (int i = 0; i < nrows; ++i) dst[(size_t)(row0 + i) * g.N + col + lane] = stg[i * kStgStride + lane];
        __syncwarp();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty_bar(buf));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// The same weight gradients on CTA pairs (cta_group::2): 256 x 256 tiles of D[e], each CTA holding
// 128 of the m rows (its A^T half) and 128 of the n columns (its B half), with stages of 128
// contraction rows.  Both CTAs' loads of a stage complete on the leader's full barrier, which the
// leader arms with both halves' bytes, and the leader issues the pair's MMAs once it completes.  A
// segment's ragged last stage runs only the 16-row MMA steps that hold segment rows; the leader's MMA
// warp first zeroes the rows past the segment inside the last of those steps, in its own shared memory
// and (through the cluster window) in the peer's.  Commits free the stage (and hand the accumulator to
// the epilogue) in both CTAs at once.
struct WgPairCfg {
  static constexpr int kTileM = 256, kTileN = 256, kStageK = 128;
  static constexpr int kStages = 3;
  static constexpr int kBoxBytes = 64 * kStageK * 2;  // one 64 (m or n) x 128 (k) box: 16 KB
  static constexpr int kABytes = 2 * kBoxBytes;        // this CTA's 128 m values
  static constexpr int kBBytes = 2 * kBoxBytes;        // this CTA's 128 n values
  static constexpr int kStageBytes = kABytes + kBBytes;  // 64 KB per CTA
  static constexpr int kTmemCols = 2 * kTileN;
  static constexpr int kBarOff = kStages * kStageBytes;
  static constexpr int kNumBars = 2 * kStages + 4 + 1;  // full, empty; tfull x2, tempty x2; drain
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kOffsOff = kMiscOff + 16;
  static constexpr int kStgOff = (kOffsOff + 260 * 4 + 1023) & ~1023;
  static constexpr int kSmemBytes = 1024 + kStgOff + kEpiWarps * kStgWarpBytes;
  static_assert(kStgOff % 16 == 0 && kSmemBytes <= 232448, "shared-memory plan");
  // kind::f16, D fp32, A and B bf16 MN-major, N = 256, M = 256 over the pair
  static constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) |
                                     ((uint32_t)(kTileN >> 3) << 17) | ((uint32_t)(kTileM >> 4) << 24);
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    wgrad_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const __grid_constant__ CUtensorMap tmD, WgradArgs g) {
  using C = WgPairCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + C::kBarOff;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (C::kStages + s); };
  auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * C::kStages + b); };
  auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * C::kStages + 2 + b); };
  const uint32_t drain_bar = bar0 + 8u * (2 * C::kStages + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);
  int* offs = reinterpret_cast<int*>(smem + C::kOffsOff);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* stg = reinterpret_cast<float*>(smem + C::kStgOff + (warp >= 2 ? warp - 2 : 0) * kStgWarpBytes);
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cluster_id = blockIdx.x >> 1, nclusters = gridDim.x >> 1;
  const int E = g.E;
  const int MT = (g.M + C::kTileM - 1) / C::kTileM, NT = (g.N + C::kTileN - 1) / C::kTileN;
  const int per_e = MT * NT;
  const int total = E * per_e;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), 2 * kEpiWarps);  // every epilogue warp of both CTAs
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  for (int i = threadIdx.x; i <= E; i += kThreads) offs[i] = g.offsets[i];
  if (warp == 1) tmem_alloc_pair(smem_u32(tmem_slot), C::kTmemCols);
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers exist before any cross-CTA signal
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  auto decode = [&](int tile, int& e, int& m0, int& n0) {
    e = tile / per_e;
    const int local = tile - e * per_e;
    n0 = (local / MT) * C::kTileN;
    m0 = (local % MT) * C::kTileM;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs) -----
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int armed[C::kStages];
      for (int s = 0; s < C::kStages; ++s) armed[s] = -1;
      bool ok = true;
      for (int tile = cluster_id; tile < total && ok; tile += nclusters) {
        int e, m0, n0;
        decode(tile, e, m0, n0);
        const int r0 = offs[e], cnt = offs[e + 1] - r0, KB = (cnt + C::kStageK - 1) / C::kStageK;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, g.wait_limit, abort_flag, g.status, kDevTimeoutProducer)) {
            ok = false;
            break;
          }
          const uint32_t a_dst = sbase + stage * C::kStageBytes;
          const uint32_t b_dst = a_dst + C::kABytes;
          const int k0 = r0 + kb * C::kStageK;
          // both CTAs' bytes complete on the leader's full barrier, which the leader arms; rows of a
          // ragged last stage past the segment are zeroed by the leader's MMA warp once they land
          if (leader) {
            mbar_arrive_expect_tx(full_bar(stage), 2 * C::kStageBytes);
            armed[stage] = (int)phase;
          }
          const uint32_t fb = peer_addr(full_bar(stage), 0);
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            tma_load_2d_pair(a_dst + j * C::kBoxBytes, &tmA, m0 + 128 * (int)rank + 64 * j, k0, fb);
            tma_load_2d_pair(b_dst + j * C::kBoxBytes, &tmB, n0 + 128 * (int)rank + 64 * j, k0, fb);
          }
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok || *abort_flag) {
        for (int s = 0; s < C::kStages; ++s)
          if (armed[s] >= 0) {
            volatile int dummy = 0;
            mbar_wait(full_bar(s), (uint32_t)armed[s], g.wait_limit, &dummy, g.status, kDevTimeoutDrain);
          }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA (leader) ---------------
    if (leader) {
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      bool issued = false;
      for (int tile = cluster_id; tile < total && ok; tile += nclusters, ++it) {
        int e, m0, n0;
        decode(tile, e, m0, n0);
        const int r0 = offs[e], cnt = offs[e + 1] - r0, KB = (cnt + C::kStageK - 1) / C::kStageK;
        const int buf = it & 1;
        const uint32_t tphase = (uint32_t)((it >> 1) & 1);
        if (!__all_sync(0xffffffffu, mbar_wait(tempty_bar(buf), tphase ^ 1u, g.wait_limit, abort_flag, g.status,
                                               kDevTimeoutMma))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(buf * C::kTileN);
        for (int kb = 0; kb < KB; ++kb) {
          if (!__all_sync(0xffffffffu, mbar_wait(full_bar(stage), phase, g.wait_limit, abort_flag, g.status,
                                                 kDevTimeoutMma))) {
            ok = false;
            break;
          }
          const uint32_t a_addr = sbase + stage * C::kStageBytes;
          const int valid = min(C::kStageK, cnt - kb * C::kStageK);
          // a ragged last stage runs only the 16-row MMA steps that hold segment rows; the rows past the
          // segment inside the last of them are zeroed first, in this CTA's four boxes and the peer's
          // (whole 128-byte lines, which the swizzle leaves in place)
          const int nk = (valid + 15) / 16;
          if (valid < 16 * nk) {
            const int per_box = (16 * nk - valid) * 8;  // 16-byte pieces per box
            for (int i = lane; i < 8 * per_box; i += 32) {
              const int box = (i / per_box) & 3, rem = i % per_box;
              const uint32_t addr = a_addr + box * C::kBoxBytes + (valid + rem / 8) * 128 + (rem % 8) * 16;
              if (i < 4 * per_box) asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};\n" ::"r"(addr), "r"(0u) : "memory");
              else asm volatile("st.shared::cluster.v4.u32 [%0], {%1, %1, %1, %1};\n" ::"r"(peer_addr(addr, 1)), "r"(0u) : "memory");
            }
            asm volatile("fence.proxy.async.shared::cluster;\n" ::: "memory");
          }
          __syncwarp();
          tc_fence_after();
          if (lane == 0) {
            const uint32_t b_addr = a_addr + C::kABytes;
            if (nk == C::kStageK / 16) {
#pragma unroll
              for (int kk = 0; kk < C::kStageK / 16; ++kk)
                mma_bf16_pair(d_tmem, desc_mnmajor(a_addr + kk * 16 * 128, C::kBoxBytes),
                              desc_mnmajor(b_addr + kk * 16 * 128, C::kBoxBytes), C::kIdesc, (kb | kk) != 0 ? 1u : 0u);
            } else {
              for (int kk = 0; kk < nk; ++kk)
                mma_bf16_pair(d_tmem, desc_mnmajor(a_addr + kk * 16 * 128, C::kBoxBytes),
                              desc_mnmajor(b_addr + kk * 16 * 128, C::kBoxBytes), C::kIdesc, (kb | kk) != 0 ? 1u : 0u);
            }
            mma_commit_both(empty_bar(stage));  // frees this stage in both CTAs once its MMAs are done
          }
          issued = true;
          __syncwarp();
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if (lane == 0) mma_commit_both(tfull_bar(buf));  // with no rows this arrives at once
        __syncwarp();
      }
      if ((!ok || *abort_flag) && issued && lane == 0) {
        mma_commit_pair(drain_bar);
        volatile int dummy = 0;
        mbar_wait(drain_bar, 0, g.wait_limit, &dummy, g.status, kDevTimeoutDrain);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..5, both) --
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;
    const uint32_t tempty_leader0 = peer_addr(tempty_bar(0), 0);
    const uint32_t tempty_leader1 = peer_addr(tempty_bar(1), 0);
    int it = 0;
    for (int tile = cluster_id; tile < total; tile += nclusters, ++it) {
      int e, m0, n0;
      decode(tile, e, m0, n0);
      const bool empty = offs[e + 1] == offs[e];
      const int buf = it & 1;
      const uint32_t tphase = (uint32_t)((it >> 1) & 1);
      const bool got = mbar_wait(tfull_bar(buf), tphase, g.wait_limit, abort_flag, g.status, kDevTimeoutEpilogue);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const int row0 = m0 + 128 * (int)rank + quarter * 32;  // this warp's 32 rows of D
      constexpr int kChunks = C::kTileN / 32 / (kEpiWarps / 4);
      uint8_t* box = reinterpret_cast<uint8_t*>(stg);  // 32 x 32 fp32, 128-byte rows, 128-byte swizzle
#pragma unroll 1
      for (int c = half * kChunks; c < (half + 1) * kChunks; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(buf * C::kTileN + c * 32), r);
        const int col = n0 + c * 32;
        if (row0 >= g.M || col >= g.N) continue;  // wholly past the edge (partial parts are clipped)
        if (lane == 0) bulk_wait_read0();  // the previous box has left the staging buffer
        __syncwarp();
        uint8_t* row = box + lane * 128;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const uint4 v = empty ? make_uint4(0u, 0u, 0u, 0u) : make_uint4(r[4 * q], r[4 * q + 1], r[4 * q + 2], r[4 * q + 3]);
          *reinterpret_cast<uint4*>(row + ((q ^ (lane & 7)) * 16)) = v;
        }
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_3d(&tmD, smem_u32(box), col, row0, e);  // rows >= M and columns >= N are not written
          bulk_commit();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(buf ? tempty_leader1 : tempty_leader0);
    }
    if (lane == 0) bulk_wait0();  // this warp's boxes are written before exit
  }

  tc_fence_before();
  __syncthreads();
  __syncwarp();
  cluster_sync_all();  // neither CTA frees TMEM or exits while the pair still uses it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, C::kTmemCols);
  }
}

// The tensor-core epilogues' activation and its derivative on given values: out[i] = act(u[i]),
// out[n + i] = act'(u[i]) (GELU or SiLU), for tests of the epilogue arithmetic.
__global__ void activation_probe_kernel(int silu_act, const float* u, float* out, long long n) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const float v = u[i];
    out[i] = silu_act ? silu(v) : gelu_erf(v);
    out[n + i] = silu_act ? silu_grad(v) : gelu_grad(v);
  }
}

// One thread waits on a barrier that nothing completes; the bound must end it.
__global__ void timeout_probe_kernel(int32_t* status, long long limit) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&bar), 1);
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    mbar_wait(smem_u32(&bar), 0, limit, &abort_flag, status, kDevTimeoutProbe);
  }
}

// ------------------------------------------------------------------ host side -------------------
PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// CTA-pair tiles are used for N divisible by 256 and K by 128 when segments are long enough;
// moe_set_kernel_options(MOE_KERNEL_NO_CTA_PAIR) selects the single-CTA kernel everywhere (for
// comparisons).
bool pair_mode_enabled() { return (kernel_options() & MOE_KERNEL_NO_CTA_PAIR) == 0; }

// A operand: [rows, K] bf16 row-major; box = 64 k x 128 rows
bool make_map_a(CUtensorMap* m, const void* base, int rows, int K) {
  auto enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)K * 2};
  cuuint32_t box[2] = {BK, BM};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A operand in boxes of box_rows rows (box = 64 k x box_rows): 16 for segments of a few rows, 8 for
// the spread placement of mid-length segments
bool make_map_a_rows(CUtensorMap* m, const void* base, int rows, int K, int box_rows) {
  auto enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)K * 2};
  cuuint32_t box[2] = {BK, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// GEMM1 output h: [rows, N] bf16 row-major; stores of 64 columns x 32 rows, 128-byte swizzle
bool make_map_store(CUtensorMap* m, void* base, int rows, int N) {
  auto enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)N, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)N * 2};
  cuuint32_t box[2] = {64, 32};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// B operand: [E, K, N] bf16 (n contiguous); box = 64 n x 64 k x 1 expert
bool make_map_b(CUtensorMap* m, const void* base, int E, int K, int N) {
  auto enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)N, (cuuint64_t)K, (cuuint64_t)E};
  cuuint64_t strides[2] = {(cuuint64_t)N * 2, (cuuint64_t)K * N * 2};
  cuuint32_t box[3] = {64, BK, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// K-major B operand: W stored [E][N][K] (k contiguous); box = 64 k x box_rows n x 1 expert
bool make_map_bk(CUtensorMap* m, const void* base, int E, int N, int K, int box_rows) {
  auto enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)K, (cuuint64_t)N, (cuuint64_t)E};
  cuuint64_t strides[2] = {(cuuint64_t)K * 2, (cuuint64_t)N * K * 2};
  cuuint32_t box[3] = {BK, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// MN-major operand of the weight gradients: [rows, C] bf16 row-major; box = 64 columns x box_rows rows
bool make_map_rows(CUtensorMap* m, const void* base, int rows, int C, int box_rows) {
  auto enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)C, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)C * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Weight-gradient output D[E][M][N] fp32; stores of 32 columns x 32 rows, 128-byte swizzle.  Three
// dimensions so that rows past M (or columns past N) of a partial tile are clipped, never written
// into the next expert.
bool make_map_dw(CUtensorMap* m, float* base, int E, int M, int N) {
  auto enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)N, (cuuint64_t)M, (cuuint64_t)E};
  cuuint64_t strides[2] = {(cuuint64_t)N * 4, (cuuint64_t)M * N * 4};
  cuuint32_t box[3] = {32, 32, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// ma16: the same A operand in 16-row boxes, used when g.a_box_rows = 16 (else any valid map)
template <int BN, int EPI, bool BKM = false>
cudaError_t launch_one(const CUtensorMap& ma, const CUtensorMap& mb, const GemmArgs& g, int grid, cudaStream_t st,
                       const CUtensorMap* ma16 = nullptr) {
  auto kern = grouped_gemm_kernel<BN, EPI, BKM>;
  cudaError_t err = ensure_smem_limit(reinterpret_cast<const void*>(kern), Cfg<BN>::kSmemBytes);
  if (err != cudaSuccess) return err;
  kern<<<grid, kThreads, Cfg<BN>::kSmemBytes, st>>>(ma, mb, ma16 ? *ma16 : ma, g);
  return cudaGetLastError();
}

template <int EPI, bool BKM = false>
cudaError_t launch_pair(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& mc, const GemmArgs& g, int grid,
                        cudaStream_t st) {
  auto kern = grouped_gemm_pair_kernel<EPI, BKM>;
  cudaError_t err = ensure_smem_limit(reinterpret_cast<const void*>(kern), PairCfg::kSmemBytes);
  if (err != cudaSuccess) return err;
  kern<<<grid & ~1, kThreads, PairCfg::kSmemBytes, st>>>(ma, mb, mc, g);
  return cudaGetLastError();
}

// 256-row CTA-pair tiles pay off when experts hold at least a full pair tile on average; with
// shorter segments (many experts, or few tokens) most of a 256-row tile would be padding, and the
// 128-row single-CTA tiles waste half as much.  The host sees only the expected rows per expert
// (T*k/E); the actual counts stay on the device.
// Small segments (a few rows per expert, e.g. decode): the GEMM streams the weights, and every tile
// loads only the 16-row A boxes that hold its rows.  The widest tile that divides N streams best:
// the longer contiguous run of each weight row outweighs a ragged last wave (decode's GEMM1 at
// 256-wide tiles, 3.03 waves, beat 128-wide, 6.05 waves; 64-wide was far slower).
int pick_bn_small(int N) { return N % 256 == 0 ? 256 : (N % 128 == 0 ? 128 : 64); }

// Whether a grouped GEMM with N output columns, contraction K and avg_rows rows per expert runs on
// CTA pairs (256 x 256 tiles) rather than single-CTA tiles.
bool pair_tiles_fit(int N, int K, long long avg_rows) {
  return N % 256 == 0 && K % PairCfg::kStageK == 0 && avg_rows >= PairCfg::kTileM && pair_mode_enabled();
}

template <int EPI>
cudaError_t launch_bn(int N, const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& mc, const GemmArgs& g,
                      int grid, long long avg_rows, cudaStream_t st, const CUtensorMap* ma16 = nullptr) {
  if (pair_tiles_fit(N, g.K, avg_rows)) return launch_pair<EPI>(ma, mb, mc, g, grid, st);
  if (ma16 != nullptr && g.a_box_rows > 0 && !g.spread_rows) {
    const int bn = pick_bn_small(N);
    if (bn == 256) return launch_one<256, EPI>(ma, mb, g, grid, st, ma16);
    if (bn == 128) return launch_one<128, EPI>(ma, mb, g, grid, st, ma16);
    return launch_one<64, EPI>(ma, mb, g, grid, st, ma16);
  }
  if (N % 256 == 0) return launch_one<256, EPI>(ma, mb, g, grid, st, ma16);
  if (N % 128 == 0) return launch_one<128, EPI>(ma, mb, g, grid, st, ma16);
  return launch_one<64, EPI>(ma, mb, g, grid, st, ma16);
}

// A [rows, K] . W[e]^T with W stored [E][N][K]: the backward's data-gradient GEMMs.
template <int EPI>
cudaError_t launch_dgrad(const void* A, int rows_cap, const void* W, int E, int N, int K, const GemmArgs& g, int grid,
                         long long avg_rows, cudaStream_t st) {
  CUtensorMap ma, mb;
  if (!make_map_a(&ma, A, rows_cap, K)) return cudaErrorInvalidValue;
  if (pair_tiles_fit(N, K, avg_rows)) {
    if (!make_map_bk(&mb, W, E, N, K, PairCfg::kHalfN)) return cudaErrorInvalidValue;
    return launch_pair<EPI, true>(ma, mb, ma, g, grid, st);
  }
  const int BN = N % 256 == 0 ? 256 : (N % 128 == 0 ? 128 : 64);
  if (!make_map_bk(&mb, W, E, N, K, BN)) return cudaErrorInvalidValue;
  if (BN == 256) return launch_one<256, EPI, true>(ma, mb, g, grid, st);
  if (BN == 128) return launch_one<128, EPI, true>(ma, mb, g, grid, st);
  return launch_one<64, EPI, true>(ma, mb, g, grid, st);
}

cudaError_t launch_wgrad(const void* A, const void* B, int rows_cap, int M, int N, const int32_t* offsets, int E,
                         float* out, int32_t* status, long long wait_limit, int grid, cudaStream_t st) {
  const bool pair = pair_mode_enabled();
  const int box_rows = pair ? WgPairCfg::kStageK : WgCfg::kBK;
  CUtensorMap ma, mb;
  if (!make_map_rows(&ma, A, rows_cap, M, box_rows) || !make_map_rows(&mb, B, rows_cap, N, box_rows))
    return cudaErrorInvalidValue;
  WgradArgs g{};
  g.offsets = offsets;
  g.E = E;
  g.M = M;
  g.N = N;
  g.out = out;
  g.status = status;
  g.wait_limit = wait_limit;
  if (pair) {
    CUtensorMap md;
    if (!make_map_dw(&md, out, E, M, N)) return cudaErrorInvalidValue;
    cudaError_t err = ensure_smem_limit(reinterpret_cast<const void*>(wgrad_pair_kernel), WgPairCfg::kSmemBytes);
    if (err != cudaSuccess) return err;
    wgrad_pair_kernel<<<grid & ~1, kThreads, WgPairCfg::kSmemBytes, st>>>(ma, mb, md, g);
    return cudaGetLastError();
  }
  cudaError_t err = ensure_smem_limit(reinterpret_cast<const void*>(wgrad_kernel), WgCfg::kSmemBytes);
  if (err != cudaSuccess) return err;
  wgrad_kernel<<<grid, kThreads, WgCfg::kSmemBytes, st>>>(ma, mb, g);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bwd_gemms_sm100(const BwdGemmArgs& a, cudaStream_t st, int* launches) {
  const int grid = a.num_sms > 0 ? a.num_sms : 148;
  // G = dout_rows . W2[e]^T (W2 stored [E][F][H]: N = F, K = H); epilogue -> du, dw partials
  GemmArgs g{};
  g.offsets = a.offsets;
  g.E = a.E;
  g.N = a.F;
  g.K = a.H;
  g.h_out = reinterpret_cast<__nv_bfloat16*>(a.du);
  g.h_in = reinterpret_cast<const __nv_bfloat16*>(a.h);
  g.u_in = reinterpret_cast<const __nv_bfloat16*>(a.u);
  g.dwraw = a.dwraw;
  g.row_token = a.row_token;
  g.row_slot = a.row_slot;
  g.topk_w = a.topk_w;
  g.k = a.k;
  g.status = a.status;
  g.wait_limit = a.wait_limit;
  cudaError_t err = a.act == MOE_ACT_SILU
                        ? launch_dgrad<EPI_DGRAD_SILU>(a.dperm, a.rows_cap, a.W2, a.E, a.F, a.H, g, grid, a.avg_rows, st)
                        : launch_dgrad<EPI_DGRAD_GELU>(a.dperm, a.rows_cap, a.W2, a.E, a.F, a.H, g, grid, a.avg_rows, st);
  if (err != cudaSuccess) return err;
  ++*launches;
  // dx[t] += du . W1[e]^T (W1 stored [E][H][F]: N = H, K = F), scatter-added with weight 1
  GemmArgs g2{};
  g2.offsets = a.offsets;
  g2.E = a.E;
  g2.N = a.H;
  g2.K = a.F;
  g2.out = a.dx;
  g2.row_token = a.row_token;
  g2.row_slot = a.row_slot;
  g2.topk_w = nullptr;
  g2.k = a.k;
  g2.status = a.status;
  g2.wait_limit = a.wait_limit;
  err = launch_dgrad<EPI_COMBINE>(a.du, a.rows_cap, a.W1, a.E, a.H, a.F, g2, grid, a.avg_rows, st);
  if (err != cudaSuccess) return err;
  ++*launches;
  // dW2[e] = h_e^T . (w dout)_e  (F x H);  dW1[e] = x_e^T . du_e  (H x F)
  err = launch_wgrad(a.h, a.dyperm, a.rows_cap, a.F, a.H, a.offsets, a.E, a.dW2, a.status, a.wait_limit, grid, st);
  if (err != cudaSuccess) return err;
  ++*launches;
  err = launch_wgrad(a.x_perm, a.du, a.rows_cap, a.H, a.F, a.offsets, a.E, a.dW1, a.status, a.wait_limit, grid, st);
  if (err != cudaSuccess) return err;
  ++*launches;
  return cudaSuccess;
}

bool ffn_gemm1_on_pairs(int H, int F, long long avg_rows) { return pair_tiles_fit(F, H, avg_rows); }

cudaError_t launch_ffn_bf16_sm100(const FfnArgs& a, cudaStream_t st, int* launches) {
  CUtensorMap ma1, mb1, ma2, mb2, mc1;
  if (!make_map_a(&ma1, a.x_perm, a.rows_cap, a.H) || !make_map_b(&mb1, a.W1, a.E, a.H, a.F) ||
      !make_map_a(&ma2, a.h, a.rows_cap, a.F) || !make_map_b(&mb2, a.W2, a.E, a.F, a.H) ||
      !make_map_store(&mc1, a.h, a.rows_cap, a.F))
    return cudaErrorInvalidValue;
  const int grid = a.num_sms > 0 ? a.num_sms : 148;
  // a few rows per expert on average (decode-sized batches): 16-row A boxes, and the tile width chosen
  // for the fewest weight-streaming waves.  (At the Switch shape's ~64 rows per expert this mode measured
  // slower: its narrower GEMM2 tiles read shorter runs of each weight row.)
  const bool small = a.avg_rows < 32;
  // 32 .. 127 rows per expert on average (the Switch shape: ~64): a tile holds one short segment, and
  // its rows are spread over all four TMEM lane quarters in 8-row groups, so that every epilogue warp
  // (and every SM sub-partition) shares the bias + activation work instead of two of the four
  const bool spread = !small && a.avg_rows < BM;
  const int box_rows = small ? 16 : 8;
  CUtensorMap ma1s, ma2s;
  if ((small || spread) && (!make_map_a_rows(&ma1s, a.x_perm, a.rows_cap, a.H, box_rows) ||
                            !make_map_a_rows(&ma2s, a.h, a.rows_cap, a.F, box_rows)))
    return cudaErrorInvalidValue;

  GemmArgs g1{};
  g1.offsets = a.offsets;
  g1.E = a.E;
  g1.N = a.F;
  g1.K = a.H;
  g1.bias = reinterpret_cast<const __nv_bfloat16*>(a.b1);
  g1.h_out = reinterpret_cast<__nv_bfloat16*>(a.h);
  g1.u_out = reinterpret_cast<__nv_bfloat16*>(a.u_out);
  g1.k = a.k;
  g1.a_box_rows = small ? 16 : (spread ? 8 : 0);
  g1.spread_rows = spread ? 1 : 0;
  g1.status = a.status;
  g1.wait_limit = a.wait_limit;
  if (a.clear_out != nullptr) {
    if (ffn_gemm1_on_pairs(a.H, a.F, a.avg_rows)) {
      g1.clear = reinterpret_cast<float4*>(a.clear_out);
      g1.clear_n = (long long)a.T * a.H / 4;
    } else {
      // only the CTA-pair GEMM1 zeroes out; callers ask for it only then, but out must hold zeros
      // before GEMM2 whichever kernel runs
      const cudaError_t e = cudaMemsetAsync(a.clear_out, 0, (size_t)a.T * a.H * sizeof(float), st);
      if (e != cudaSuccess) return e;
    }
  }
  const long long avg_rows = a.avg_rows;
  cudaError_t err = a.act == MOE_ACT_SILU
                        ? launch_bn<EPI_SILU>(a.F, ma1, mb1, mc1, g1, grid, avg_rows, st, (small || spread) ? &ma1s : nullptr)
                        : launch_bn<EPI_GELU>(a.F, ma1, mb1, mc1, g1, grid, avg_rows, st, (small || spread) ? &ma1s : nullptr);
  if (err != cudaSuccess) return err;
  ++*launches;

  GemmArgs g2 = g1;
  g2.clear = nullptr;
  g2.clear_n = 0;
  g2.N = a.H;
  g2.K = a.F;
  g2.bias = reinterpret_cast<const __nv_bfloat16*>(a.b2);
  g2.h_out = nullptr;
  g2.u_out = nullptr;
  g2.out = a.out;
  g2.y = a.y;
  g2.row_token = a.row_token;
  g2.row_slot = a.row_slot;
  g2.topk_w = a.topk_w;
  // top-1 layers on single-CTA tiles with a long K (the Switch shape: 512 tiles of K = 4096 are 3.46
  // waves on 148 SMs): two K halves per tile even out the last wave; with one slot per token each
  // element of out still receives a fixed pair of adds
  const bool pair2 = pair_tiles_fit(a.H, a.F, avg_rows);
  if (a.fuse_combine && a.k == 1 && !small && !pair2 && a.F / BK >= 32) g2.k_splits = 2;
  if (a.fuse_combine)
    err = launch_bn<EPI_COMBINE>(a.H, ma2, mb2, ma2, g2, grid, avg_rows, st, (small || spread) ? &ma2s : nullptr);
  else
    err = launch_bn<EPI_STORE_Y>(a.H, ma2, mb2, ma2, g2, grid, avg_rows, st, (small || spread) ? &ma2s : nullptr);
  if (err != cudaSuccess) return err;
  ++*launches;
  return cudaSuccess;
}

// logits[T,E] (fp32) = x[T,H] . Wg[H,E] + bg on the tensor cores: one dense segment through the
// single-CTA kernel with 128 x 64 tiles and the fp32 store epilogue (bias added there).
cudaError_t launch_gate_logits_sm100(const void* x, const void* Wg, const void* bg, int T, int H, int E, float* logits,
                                     int32_t* status, long long wait_limit, int num_sms, cudaStream_t st) {
  CUtensorMap ma, mb;
  if (!make_map_a(&ma, x, T, H) || !make_map_b(&mb, Wg, 1, H, E)) return cudaErrorInvalidValue;
  GemmArgs g{};
  g.offsets = nullptr;
  g.single_rows = T;
  g.E = 1;
  g.N = E;
  g.K = H;
  g.bias = reinterpret_cast<const __nv_bfloat16*>(bg);
  g.y = logits;
  g.status = status;
  g.wait_limit = wait_limit;
  const int tiles = ((T + BM - 1) / BM) * (E / 64);
  const int grid = tiles < num_sms ? tiles : num_sms;
  return launch_one<64, EPI_STORE_Y>(ma, mb, g, grid, st);
}

// The whole gate of a bf16 layer with E = 64, 128 or 256 experts in one launch: logits = x.Wg + bg
// on the tensor cores (128-token x E tiles, one dense segment) and, in the epilogue, the softmax,
// top-k, renormalised weights, per-chunk loss partials and per-slot chunk histograms.
cudaError_t launch_gate_router_sm100(const RouterArgs& a, cudaStream_t st) {
  CUtensorMap ma, mb;
  if (!make_map_a(&ma, a.x, a.T, a.H) || !make_map_b(&mb, a.Wg, 1, a.H, a.E)) return cudaErrorInvalidValue;
  GemmArgs g{};
  g.offsets = nullptr;
  g.single_rows = a.T;
  g.E = 1;
  g.N = a.E;
  g.K = a.H;
  g.k = a.k;
  g.bias = reinterpret_cast<const __nv_bfloat16*>(a.bg);
  g.r_topk_idx = a.topk_idx;
  g.r_topk_w = a.topk_w;
  g.r_loss_part = a.loss_part;
  g.r_chunk_hist = a.chunk_hist;
  g.r_logits = a.logits_out;
  g.status = a.status;
  g.wait_limit = a.wait_limit;
  const int tiles = (a.T + BM - 1) / BM;
  const int sms = a.num_sms > 0 ? a.num_sms : 148;
  const int grid = tiles < sms ? tiles : sms;
  if (a.E == 64) return launch_one<64, EPI_ROUTER>(ma, mb, g, grid, st);
  if (a.E == 128) return launch_one<128, EPI_ROUTER>(ma, mb, g, grid, st);
  if (a.E == 256) return launch_one<256, EPI_ROUTER>(ma, mb, g, grid, st);
  return cudaErrorInvalidValue;
}

cudaError_t launch_activation_probe(int act, const float* u, float* out, long long n, cudaStream_t st) {
  const long long blocks = (n + 255) / 256;
  activation_probe_kernel<<<(int)(blocks < 1024 ? (blocks > 0 ? blocks : 1) : 1024), 256, 0, st>>>(
      act == MOE_ACT_SILU ? 1 : 0, u, out, n);
  return cudaGetLastError();
}

cudaError_t launch_timeout_probe(int32_t* status, long long limit, cudaStream_t st) {
  timeout_probe_kernel<<<1, 32, 0, st>>>(status, limit);
  return cudaGetLastError();
}

}  // namespace moe

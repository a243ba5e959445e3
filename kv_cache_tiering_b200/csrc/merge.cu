// Exact log-sum-exp merge of split partials ("Context beyond VRAM", section "What I
// built": the tiers are merged with exact attention arithmetic).
//
// One CTA of 256 threads per (sequence, query head).  The slots of the sequence are taken
// in chunks of up to kChunk:
//   1. M = max of the chunk's LSE values joined with the running maximum;
//   2. w_s = exp(LSE_s - M) into shared memory, their sum L;
//   3. warp w accumulates slots w, w + 8, ... of the chunk, lane l owning coordinates
//      [P*l, P*l + P) (coalesced rows), and the eight warp sums are added in warp order.
// Partial sums from an earlier chunk are rescaled by exp(M_old - M_new).  Every sum is taken
// in a fixed order, so the result is deterministic.  The kernel is bound by memory latency
// (a few KB per CTA), so each thread's LSE values and each warp's first kRows partial rows of
// a chunk are requested together, before the first reduction, and later rows kRows at a time.
#include "akv_internal.cuh"

namespace akv {
namespace {

constexpr int kMergeThreads = 256;
constexpr int kMergeWarps = kMergeThreads / 32;
constexpr int kChunk = 1024;

__device__ __forceinline__ float block_max(float v, float* red) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float m = red[0];
#pragma unroll
  for (int w = 1; w < kMergeWarps; ++w) m = fmaxf(m, red[w]);
  return m;
}

__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float s = red[0];
#pragma unroll
  for (int w = 1; w < kMergeWarps; ++w) s += red[w];
  return s;
}

template <int D>
__global__ void __launch_bounds__(kMergeThreads) merge_kernel(const __grid_constant__ MergeParams p) {
  constexpr int P = D / 32;                          // coordinates per lane
  constexpr int kPer = kChunk / kMergeThreads;       // LSE values per thread in a chunk
  constexpr int kRows = 8;                           // partial rows in flight per warp
  __shared__ float wsh[kChunk];
  __shared__ float red[kMergeWarps];
  __shared__ float acc_sh[kMergeWarps][D];
  const int bl = blockIdx.x, h = blockIdx.y;
  const int b = p.b0 + bl;
  const int base = p.slot_base[bl], n = p.n_slots[bl];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  allow_next_grid();
  wait_prior_grids();  // the partials come from the attention launches before this one

  float M = -INFINITY, L = 0.f;
  float acc[P];
#pragma unroll
  for (int j = 0; j < P; ++j) acc[j] = 0.f;
  // rows of slots c0 + r0 + warp + kMergeWarps i (i < kRows) that lie below cn; zeros past it
  float rows[kRows][P];
  auto load_rows = [&](int c0, int r0, int cn) {
#pragma unroll
    for (int i = 0; i < kRows; ++i) {
      const int s = r0 + warp + kMergeWarps * i;
#pragma unroll
      for (int j = 0; j < P; ++j) rows[i][j] = 0.f;
      if (s < cn) {
        const float* row = p.o_part + ((size_t)(base + c0 + s) * p.Hq + h) * D + P * lane;
        if constexpr (P == 4) {
          const float4 v = __ldcg(reinterpret_cast<const float4*>(row));
          rows[i][0] = v.x; rows[i][1] = v.y; rows[i][2] = v.z; rows[i][3] = v.w;
        } else {
          const float2 v = __ldcg(reinterpret_cast<const float2*>(row));
          rows[i][0] = v.x; rows[i][1] = v.y;
        }
      }
    }
  };

  for (int c0 = 0; c0 < n; c0 += kChunk) {
    const int cn = min(kChunk, n - c0);
    float ls[kPer];
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
      const int s = (int)threadIdx.x + kMergeThreads * k;
      ls[k] = s < cn ? __ldcg(p.lse_part + (size_t)(base + c0 + s) * p.Hq + h) : -INFINITY;
    }
    load_rows(c0, 0, cn);
    float m = -INFINITY;
#pragma unroll
    for (int k = 0; k < kPer; ++k) m = fmaxf(m, ls[k]);
    const float M_new = fmaxf(M, block_max(m, red));
    if (M_new == -INFINITY) continue;  // nothing finite so far
    const float r = expf(M - M_new);   // 0 while M is -inf
    float part = 0.f;
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
      const int s = (int)threadIdx.x + kMergeThreads * k;
      if (s < cn) {
        const float w = expf(ls[k] - M_new);
        wsh[s] = w;
        part += w;
      }
    }
    L = L * r + block_sum(part, red);  // block_sum's barriers also publish wsh
#pragma unroll
    for (int j = 0; j < P; ++j) acc[j] *= r;
    for (int r0 = 0; r0 < cn; r0 += kMergeWarps * kRows) {
      if (r0 > 0) load_rows(c0, r0, cn);
#pragma unroll
      for (int i = 0; i < kRows; ++i) {
        const int s = r0 + warp + kMergeWarps * i;
        if (s < cn) {
          const float w = wsh[s];
#pragma unroll
          for (int j = 0; j < P; ++j) acc[j] = fmaf(w, rows[i][j], acc[j]);
        }
      }
    }
    M = M_new;
    __syncthreads();  // wsh is rewritten by the next chunk
  }
#pragma unroll
  for (int j = 0; j < P; ++j) acc_sh[warp][P * lane + j] = acc[j];
  __syncthreads();
  for (int i = threadIdx.x; i < D; i += kMergeThreads) {
    float o = 0.f;
    if (M != -INFINITY) {
      for (int w = 0; w < kMergeWarps; ++w) o += acc_sh[w][i];
      o /= L;
    }
    p.o[((size_t)b * p.Hq + h) * D + i] = o;
  }
  if (threadIdx.x == 0) p.lse[(size_t)b * p.Hq + h] = (M == -INFINITY) ? -INFINITY : M + logf(L);
}

}  // namespace

cudaError_t launch_merge(const MergeParams& p, int d, cudaStream_t s) {
  dim3 grid(p.n_seq, p.Hq);
  cudaError_t e = d == 128 ? launch_overlapped(merge_kernel<128>, grid, dim3(kMergeThreads), 0, s, p)
                           : launch_overlapped(merge_kernel<64>, grid, dim3(kMergeThreads), 0, s, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace akv

// Exact log-sum-exp merge of split partials ("Context beyond VRAM", section "What I
// built": the tiers are merged with exact attention arithmetic).  One CTA of D threads
// per (sequence, query head); thread i owns output coordinate i.  The partials of a
// sequence are read in increasing slot order, so the result is deterministic.
#include "akv_internal.cuh"

namespace akv {
namespace {

template <int D>
__global__ void __launch_bounds__(D) merge_kernel(const __grid_constant__ MergeParams p) {
  const int bl = blockIdx.x, h = blockIdx.y;
  const int b = p.b0 + bl;
  const int base = p.slot_base[bl], n = p.n_slots[bl];
  const int i = threadIdx.x;
  float m = -INFINITY;
  for (int s = 0; s < n; ++s) m = fmaxf(m, __ldg(p.lse_part + (size_t)(base + s) * p.Hq + h));
  float o = 0.f, l = 0.f;
  if (m != -INFINITY) {
    for (int s = 0; s < n; ++s) {
      const float ls = __ldg(p.lse_part + (size_t)(base + s) * p.Hq + h);
      const float w = expf(ls - m);  // exp(-inf) = 0 for an empty partial
      l += w;
      o = fmaf(w, __ldg(p.o_part + ((size_t)(base + s) * p.Hq + h) * D + i), o);
    }
    o /= l;
  }
  p.o[((size_t)b * p.Hq + h) * D + i] = o;
  if (i == 0) p.lse[(size_t)b * p.Hq + h] = (m == -INFINITY) ? -INFINITY : m + logf(l);
}

}  // namespace

cudaError_t launch_merge(const MergeParams& p, int d, cudaStream_t s) {
  dim3 grid(p.n_seq, p.Hq);
  if (d == 128) merge_kernel<128><<<grid, 128, 0, s>>>(p);
  else merge_kernel<64><<<grid, 64, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace akv

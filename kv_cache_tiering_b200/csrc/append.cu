// Appending the new token of a decode step: one warp copies one (sequence, KV head) key row
// and value row into the BF16 tier at the sequence's position, addressed exactly as the
// attention kernels read it (strides, or the page table of a paged tier).
#include "akv_internal.cuh"

namespace akv {
namespace {

template <int D>
__global__ void __launch_bounds__(32) append_kernel(const __grid_constant__ AppendParams p) {
  const int bl = blockIdx.x, h = blockIdx.y, lane = threadIdx.x;
  const int pos = p.pos[bl];
  if (pos < 0) return;
  const int b = p.b0 + bl;
  const TierDev& t = p.tier;
  int64_t e;  // element offset of the destination row
  if (t.paged) {
    const int32_t pg = __ldcg(t.page_table + (int64_t)b * t.pt_stride + (pos >> 4));
    if (pg < 0 || (int64_t)pg >= t.n_pages) {  // no write outside the pool
      if (lane == 0) flag_error(p.err, AKV_EFLAG_BOUNDS);
      return;
    }
    e = (int64_t)pg * t.s_seq + (int64_t)h * t.s_head + (int64_t)(pos & 15) * t.s_tok;
  } else {
    e = (int64_t)b * t.s_seq + (int64_t)h * t.s_head + (int64_t)pos * t.s_tok;
  }
  constexpr int W = D / 32;  // bf16 elements per lane
  const size_t src = ((size_t)b * p.Hkv + h) * D + (size_t)W * lane;
  uint8_t* dk = const_cast<uint8_t*>(t.k) + 2 * (e + W * lane);
  uint8_t* dv = const_cast<uint8_t*>(t.v) + 2 * (e + W * lane);
  if constexpr (W == 4) {
    *reinterpret_cast<uint2*>(dk) = *reinterpret_cast<const uint2*>(p.new_k + src);
    *reinterpret_cast<uint2*>(dv) = *reinterpret_cast<const uint2*>(p.new_v + src);
  } else {
    *reinterpret_cast<uint32_t*>(dk) = *reinterpret_cast<const uint32_t*>(p.new_k + src);
    *reinterpret_cast<uint32_t*>(dv) = *reinterpret_cast<const uint32_t*>(p.new_v + src);
  }
}

}  // namespace

cudaError_t launch_append(const AppendParams& p, int d, int n_seq, cudaStream_t s) {
  const dim3 grid(n_seq, p.Hkv);
  if (d == 128) append_kernel<128><<<grid, 32, 0, s>>>(p);
  else append_kernel<64><<<grid, 32, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace akv

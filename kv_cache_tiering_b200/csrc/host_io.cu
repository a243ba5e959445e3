// A decode step whose query and outputs live in page-locked host memory: the query is read
// over PCIe by the GPU itself into device scratch, ahead of the attention launches, so the
// whole step (copy, attention, merge) stays on one stream with launch overlap between its
// kernels.  The merge writes O and LSE straight into the host arrays.
#include "akv_internal.cuh"

namespace akv {
namespace {

constexpr int kCopyThreads = 256;
constexpr int kCopyPer = 4;  // 16-byte units per thread

struct CopyParams {
  const uint4* src;  // device address of the host array
  uint4* dst;
  int64_t n16;       // 16-byte units
};

// The host array is fixed from the call until its work completes, so it is read before the
// wait: the PCIe round trip overlaps the previous kernel on the stream, and only the writes
// (dst may still be read by the previous step's kernels) wait for it.
__global__ void __launch_bounds__(kCopyThreads) copy_in_kernel(const __grid_constant__ CopyParams p) {
  allow_next_grid();
  const int64_t i0 = ((int64_t)blockIdx.x * kCopyThreads + threadIdx.x) * kCopyPer;
  uint4 v[kCopyPer];
#pragma unroll
  for (int k = 0; k < kCopyPer; ++k)
    if (i0 + k < p.n16) v[k] = __ldcv(p.src + i0 + k);  // host memory: read it, never a cached copy
  wait_prior_grids();
#pragma unroll
  for (int k = 0; k < kCopyPer; ++k)
    if (i0 + k < p.n16) p.dst[i0 + k] = v[k];
}

}  // namespace

cudaError_t launch_copy_in(const void* src, void* dst, size_t bytes, cudaStream_t s) {
  CopyParams p;
  p.src = static_cast<const uint4*>(src);
  p.dst = static_cast<uint4*>(dst);
  p.n16 = (int64_t)(bytes / 16);
  if (p.n16 == 0) return cudaSuccess;
  const int64_t per_cta = (int64_t)kCopyThreads * kCopyPer;
  const int64_t grid = (p.n16 + per_cta - 1) / per_cta;
  if (grid > INT32_MAX) return cudaErrorInvalidValue;
  cudaError_t e = launch_overlapped(copy_in_kernel, dim3((unsigned)grid), dim3(kCopyThreads), 0, s, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace akv

// Internal declarations shared by the libakv translation units: launch-parameter
// structs (passed by value as __grid_constant__ kernel parameters, so the library needs
// no device scratch for its per-sequence tables), device helpers for BF16 / tier
// addressing, and the host-side launchers.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "../../include/akv.h"

namespace akv {

// Sequences handled by one launch; larger batches are cut into several launches.
constexpr int kMaxSeqPerLaunch = 256;
constexpr int kPageTokens = AKV_PAGE_TOKENS;
constexpr int kMaxSplitTokens = 1024;

// Device view of one tier (byte pointers; strides in elements for BF16, blocks for CODES4).
struct TierDev {
  const uint8_t* k;
  const uint8_t* v;
  const int32_t* page_table;
  int64_t pt_stride;
  int64_t n_pages;
  int64_t s_seq, s_head, s_tok;
  int32_t paged;
  uint32_t signs[4];  // CODES4: coordinate i negated before the rotation when bit i is set
};

// +1 or -1: the rotation sign of coordinate i of a compact tier.
__device__ __forceinline__ float coord_sign(const TierDev& t, int i) {
  return ((t.signs[i >> 5] >> (i & 31)) & 1u) ? -1.f : 1.f;
}

// Per-launch sequence table: work item i of the launch belongs to the sequence b with
// item_base[b] <= i < item_base[b + 1]; b is local to the launch, b0 + b is global.
struct SeqTable {
  int32_t n_seq;
  int32_t b0;
  int32_t item_base[kMaxSeqPerLaunch + 1];
  int32_t len[kMaxSeqPerLaunch];
  int32_t slot_base[kMaxSeqPerLaunch];
};

struct AttendParams {
  CUtensorMap tmk, tmv;  // TMA descriptors of a BF16 tier's K and V (tensor-core kernel)
  int8_t tperm[3];       // TMA dim j+1 takes logical coordinate tperm[j] (0 token, 1 head, 2 seq/page)
  const uint16_t* q;     // [B][Hq][D] bf16
  float* o_part;         // [n_slots][Hq][D]
  float* lse_part;       // [n_slots][Hq]
  int32_t* err;          // device error word or null
  TierDev tier;
  int32_t Hq, Hkv, split_tokens;
  float scale_log2;      // softmax_scale * log2(e): scores are kept in base-2 units
  uint16_t centroids[16];
  SeqTable seq;
};

struct EncodeParams {
  TierDev src;           // BF16 tier
  TierDev dst;           // CODES4 tier (written)
  int32_t* err;
  int32_t Hkv;
  double bound[15];      // decision boundaries (c_j + c_{j+1}) / 2, exact in float64
  SeqTable seq;          // items are 16-token blocks
};

struct AppendParams {
  TierDev tier;          // BF16 tier whose rows are written
  const uint16_t* new_k;  // [B][Hkv][D] bf16 (whole call)
  const uint16_t* new_v;
  int32_t* err;
  int32_t Hkv;
  int32_t b0;            // global index of the launch's first sequence
  int32_t pos[kMaxSeqPerLaunch];
};

struct MergeParams {
  const float* o_part;
  const float* lse_part;
  float* o;
  float* lse;
  int32_t Hq;
  int32_t n_seq, b0;
  int32_t slot_base[kMaxSeqPerLaunch];
  int32_t n_slots[kMaxSeqPerLaunch];
};

// ------------------------------------------------------------------------------------
// device helpers
// ------------------------------------------------------------------------------------

__device__ __forceinline__ int find_seq(const SeqTable& st, int item) {
  int lo = 0, hi = st.n_seq - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (st.item_base[mid] <= item) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Programmatic dependent launch.  A kernel launched with launch_overlapped may begin while
// the previous kernel on its stream finishes: it lets its own successor be scheduled early,
// does set-up that touches no global memory, then waits until the previous grid has
// completed and its writes are visible -- before its first global read or write.
__device__ __forceinline__ void allow_next_grid() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }
__device__ __forceinline__ void wait_prior_grids() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }

__device__ __forceinline__ void flag_error(int32_t* err, int32_t bits) {
  if (err) atomicOr(err, bits);
}

// Two packed bf16 -> two floats (exact).
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ float bf16_to_float(uint16_t h) { return __uint_as_float(((uint32_t)h) << 16); }

__device__ __forceinline__ float half_bits_to_float(uint16_t h) {
  return __half2float(__ushort_as_half(h));
}

// Physical page of logical page `lp` of global sequence b; out-of-pool ids are flagged
// and replaced by page 0 so no access leaves the pool.
__device__ __forceinline__ int64_t tier_page(const TierDev& t, int b, int lp, int32_t* err) {
  int32_t p = __ldcg(t.page_table + (int64_t)b * t.pt_stride + lp);
  if (p < 0 || (int64_t)p >= t.n_pages) {
    flag_error(err, AKV_EFLAG_BOUNDS);
    p = 0;
  }
  return p;
}

// Byte address of the BF16 row of token t (tier-relative), sequence b (global), KV head h.
__device__ __forceinline__ const uint8_t* bf16_row(const TierDev& t, const uint8_t* base, int b, int h,
                                                   int tok, int32_t* err) {
  int64_t e;
  if (t.paged) {
    e = tier_page(t, b, tok >> 4, err) * t.s_seq + (int64_t)h * t.s_head + (int64_t)(tok & 15) * t.s_tok;
  } else {
    e = (int64_t)b * t.s_seq + (int64_t)h * t.s_head + (int64_t)tok * t.s_tok;
  }
  return base + 2 * e;
}

// Byte address of the CODES4 block holding token t (tier-relative).
template <int D>
__device__ __forceinline__ const uint8_t* codes_block(const TierDev& t, const uint8_t* base, int b, int h,
                                                      int tok, int32_t* err) {
  constexpr int64_t BB = AKV_CODES4_BLOCK_BYTES(D);
  int64_t blk;
  if (t.paged) {
    blk = tier_page(t, b, tok >> 4, err) * t.s_seq + (int64_t)h * t.s_head;
  } else {
    blk = (int64_t)b * t.s_seq + (int64_t)h * t.s_head + (int64_t)(tok >> 4) * t.s_tok;
  }
  return base + blk * BB;
}

// ------------------------------------------------------------------------------------
// per-device launch set-up, done once
// ------------------------------------------------------------------------------------
constexpr int kMaxDevices = 64;

// Raise `Kernel`'s dynamic shared-memory limit on the current device to at least `bytes`.
// The runtime keeps the attribute, so only the first launch that needs more pays the call.
template <auto Kernel>
inline cudaError_t ensure_smem(int bytes) {
  static std::atomic<int> have[kMaxDevices];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < kMaxDevices && have[dev].load(std::memory_order_acquire) >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && dev >= 0 && dev < kMaxDevices) {
    int cur = have[dev].load(std::memory_order_relaxed);
    while (cur < bytes && !have[dev].compare_exchange_weak(cur, bytes)) {
    }
  }
  return e;
}

// Launch `kernel` so that it may overlap the tail of the previous kernel on `s` (the kernel
// must call wait_prior_grids before touching global memory).
template <typename P>
inline cudaError_t launch_overlapped(void (*kernel)(P), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                                     const P& params) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, params);
}

// Streaming multiprocessors of the current device (queried once per device).
inline int sm_count() {
  static std::atomic<int> cached[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 1;
  if (dev >= 0 && dev < kMaxDevices) {
    const int c = cached[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int n = 0;
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  n = n > 0 ? n : 1;
  if (dev >= 0 && dev < kMaxDevices) cached[dev].store(n, std::memory_order_relaxed);
  return n;
}

// ------------------------------------------------------------------------------------
// host-side launchers (return cudaGetLastError() of the launch)
// ------------------------------------------------------------------------------------

cudaError_t launch_encode(const EncodeParams& p, int d, int n_items, cudaStream_t s);
cudaError_t launch_append(const AppendParams& p, int d, int n_seq, cudaStream_t s);
cudaError_t launch_attend_simt(const AttendParams& p, int d, int G, int kind, int n_items, cudaStream_t s);
// Tensor-core split attention of one tier: a persistent grid of at most max_ctas CTAs (0: one
// per SM); overlap = launched with programmatic stream serialization.
cudaError_t launch_attend_mma(const AttendParams& p, int d, int G, int kind, int n_items, cudaStream_t s,
                              int max_ctas = 0, bool overlap = true);
// Warps per CTA of the compact-tier kernel for group size G (each runs one split at a time).
int codes_warps_per_cta(int G);
// Fill p.tmk / p.tmv for a BF16 tier of B sequences (tokens [0, max_len)): 4-D maps
// (d, tokens, heads, sequences or pages), 64-element x 16-token boxes, 128-byte swizzle.
cudaError_t make_bf16_tensor_maps(AttendParams& p, const akv_tier* t, int B, int Hkv, int d, int64_t max_len);
cudaError_t launch_merge(const MergeParams& p, int d, cudaStream_t s);
// Copy `bytes` (a multiple of 16) from host memory at device address src to dst, as a kernel
// that reads at once and waits for the previous kernel on `s` only before writing.
cudaError_t launch_copy_in(const void* src, void* dst, size_t bytes, cudaStream_t s);

// Input copy a call enqueues after its checks and before its first attention launch: a
// kernel reading mapped host memory (kernel = true) or a copy-engine transfer.
struct CopyIn {
  const void* src;
  void* dst;
  size_t bytes;
  bool kernel;
};

// Byte layout of an akv_decode workspace: LSE partials [n_slots][Hq] float, then O partials
// [n_slots][Hq][d] float, each 256-byte aligned.
struct WorkspaceLayout {
  size_t lse, o, total;
};
WorkspaceLayout workspace_layout(int B, int Hq, int Hkv, int d, int64_t n_slots);

// A checked token append of at most kMaxSeqPerLaunch sequences, not yet enqueued.
struct PendingAppend {
  AppendParams p;
  int d, n_seq;
  bool write;  // some position is >= 0 (false: nothing to enqueue)
};
// The checks and parameters of akv_append_tokens (same refusals); *single is false when the
// batch needs more than one launch, and then `out` is not filled.
akv_status prepare_append(const akv_tier* tier, const int32_t* pos, int B, int Hkv, int d, const void* new_k,
                          const void* new_v, int32_t* err_word, PendingAppend* out, bool* single);

// Validated split attention of every tier; copy_in (may be null) is enqueued after the checks
// and before the first attention launch.  append (may be null) writes a token the BF16 tier
// reads: it is enqueued before that tier's launch, on the stream that launch goes to, so when
// the tiers run side by side the append overlaps the compact tier.
akv_status attend_impl(const void* q, int B, int Hq, int Hkv, int d, float softmax_scale, const akv_tier* tiers,
                       int n_tiers, int split_tokens, float* o_part, float* lse_part, int64_t n_slots, int variant,
                       int32_t* err_word, cudaStream_t st, const CopyIn* copy_in = nullptr,
                       const PendingAppend* append = nullptr);

// Set the thread's last-error message; returns st.
akv_status set_error(akv_status st, const char* msg);

// host: the binary16 centroid table and its float64 decision boundaries
const uint16_t* centroid_table_f16();
const double* centroid_boundaries();

}  // namespace akv

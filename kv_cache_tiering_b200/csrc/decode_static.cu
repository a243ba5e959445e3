// akv_decode_static: the whole decode step for callers that cannot allocate device memory.
//
// akv_decode needs a scratch workspace for its split partials, and leaves it to the caller
// to provide one.  Some callers have no way to get device memory at the moment they decode:
// a plugin living in a process whose memory pool belongs to another framework and is not
// shared with it, or a serving loop that has frozen allocation so that no call can block on
// the allocator or synchronise the device.  This entry point serves them: its scratch is a
// fixed array in this library's device memory, so the call needs nothing beyond its inputs
// and outputs.  (It is not for code running inside a host function enqueued on a stream:
// CUDA forbids every runtime call there, and this one launches kernels.)
//
// The array is a file-scope __device__ object of AKV_DECODE_STATIC_MAX_BYTES.  Every GPU
// that loads the library holds it until the process exits.  Host code cannot use the
// array's name as a device address, so the first call on each device looks the address
// up with cudaGetSymbolAddress while that device is current, and later calls on the
// device reuse it.  Under CUDA's lazy module loading that first lookup also loads this
// library's device code on the device, which reserves the array and may block: make one
// warm-up call before freezing allocation or starting a stream capture.  All calls share
// the one array: it keeps whatever the last call left in it, and two calls whose work
// overlaps on the GPU (two streams, say) race on the array -- order them.
#include <cstdio>
#include <mutex>

#include "akv_internal.cuh"

namespace {

__device__ __align__(256) uint8_t g_decode_scratch[AKV_DECODE_STATIC_MAX_BYTES];

std::mutex g_scratch_mu;
void* g_scratch_addr[akv::kMaxDevices];  // device address of g_decode_scratch, per device

// The scratch's device address on the current device (looked up once per device).
akv_status scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return akv::set_error(AKV_ERR_CUDA, cudaGetErrorString(e));
  if (dev < 0 || dev >= akv::kMaxDevices) {
    char msg[96];
    std::snprintf(msg, sizeof(msg), "akv_decode_static: device index %d is not below %d", dev, akv::kMaxDevices);
    return akv::set_error(AKV_ERR_UNSUPPORTED, msg);
  }
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess || !p) {
      cudaGetLastError();
      return akv::set_error(AKV_ERR_CUDA, "cudaGetSymbolAddress of the static decode scratch failed");
    }
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return AKV_OK;
}

constexpr int kMaxTiers = 8;

}  // namespace

extern "C" akv_status akv_decode_static(const void* q, int B, int Hq, int Hkv, int d, float softmax_scale,
                                        const akv_tier* tiers, int n_tiers, int split_tokens, float* o, float* lse,
                                        int variant, int32_t* err_word, akv_stream_t stream) {
  if (B < 0 || B > AKV_DECODE_STATIC_MAX_SEQ)
    return akv::set_error(AKV_ERR_BUDGET, "akv_decode_static: batch outside [0, AKV_DECODE_STATIC_MAX_SEQ]");
  if (n_tiers < 0 || n_tiers > kMaxTiers) return akv::set_error(AKV_ERR_UNSUPPORTED, "akv_decode_static: 0..8 tiers");
  if (n_tiers > 0 && !tiers) return akv::set_error(AKV_ERR_INVALID, "tiers is null");
  if (Hq <= 0 || Hkv <= 0 || d <= 0) return akv::set_error(AKV_ERR_INVALID, "Hq, Hkv and d must be positive");
  if (B == 0) return AKV_OK;
  // the slot plan lives on the stack: nothing here allocates, on the device or the host
  int32_t tier_base[kMaxTiers][AKV_DECODE_STATIC_MAX_SEQ];
  int32_t seq_base[AKV_DECODE_STATIC_MAX_SEQ], seq_n[AKV_DECODE_STATIC_MAX_SEQ];
  const int32_t* lens[kMaxTiers];
  int32_t* bases[kMaxTiers];
  akv_tier planned[kMaxTiers];
  for (int i = 0; i < n_tiers; ++i) {
    if (!tiers[i].lens) return akv::set_error(AKV_ERR_INVALID, "a tier's lens is null");
    lens[i] = tiers[i].lens;
    bases[i] = tier_base[i];
    planned[i] = tiers[i];
    planned[i].slot_base = tier_base[i];
  }
  if (split_tokens < 16 || split_tokens > akv::kMaxSplitTokens || split_tokens % 16)
    return akv::set_error(AKV_ERR_UNSUPPORTED, "split_tokens must be a multiple of 16 in [16, 1024]");
  int64_t n_slots = 0;
  akv_status s = akv_plan_slots(B, n_tiers, lens, split_tokens, bases, seq_base, seq_n, &n_slots);
  if (s != AKV_OK) return s;
  const akv::WorkspaceLayout lay = akv::workspace_layout(B, Hq, Hkv, d, n_slots);
  if (lay.total > (size_t)AKV_DECODE_STATIC_MAX_BYTES)
    return akv::set_error(AKV_ERR_BUDGET,
                          "akv_decode_static: this step needs more scratch than AKV_DECODE_STATIC_MAX_BYTES; "
                          "use akv_decode with a caller-provided workspace");
  if (!o || !lse) return akv::set_error(AKV_ERR_INVALID, "o and lse must not be null");
  void* scratch = nullptr;
  if ((s = scratch_address(&scratch)) != AKV_OK) return s;
  uint8_t* ws = static_cast<uint8_t*>(scratch);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  float* lse_part = reinterpret_cast<float*>(ws + lay.lse);
  float* o_part = reinterpret_cast<float*>(ws + lay.o);
  s = akv::attend_impl(q, B, Hq, Hkv, d, softmax_scale, planned, n_tiers, split_tokens, o_part, lse_part, n_slots,
                       variant, err_word, st);
  if (s != AKV_OK) return s;
  return akv_merge_lse(o_part, lse_part, n_slots, seq_base, seq_n, B, Hq, d, o, lse, stream);
}

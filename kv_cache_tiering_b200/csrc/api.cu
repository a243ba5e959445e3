// Host side of the libakv C ABI: argument validation (nothing is launched for a refused
// call), the per-launch sequence tables, the slot planner and the staging ring.
#include <chrono>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>
#include <thread>
#include <vector>

#include <algorithm>
#include <mutex>

#include <cudaTypedefs.h>

#include "akv_internal.cuh"

namespace {

thread_local std::string g_last_error;

akv_status fail(akv_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  std::vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

akv_status ok() {
  g_last_error.clear();
  return AKV_OK;
}

akv_status cuda_fail(cudaError_t e, const char* what) {
  return fail(AKV_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

bool supported_group(int G) { return G == 1 || G == 2 || G == 4 || G == 8; }

// Validate a tier for B sequences.  need_slots: check slot ranges against n_slots.
akv_status check_tier(const akv_tier* t, int idx, int B, int d, int split_tokens, bool need_slots,
                      int64_t n_slots, int expect_kind) {
  if (!t) return fail(AKV_ERR_INVALID, "tier %d is null", idx);
  if (t->kind != AKV_TIER_BF16 && t->kind != AKV_TIER_CODES4)
    return fail(AKV_ERR_INVALID, "tier %d: unknown kind %d", idx, t->kind);
  if (expect_kind >= 0 && t->kind != expect_kind)
    return fail(AKV_ERR_INVALID, "tier %d: kind %d where %d is required", idx, t->kind, expect_kind);
  if (t->paged != 0 && t->paged != 1) return fail(AKV_ERR_INVALID, "tier %d: paged must be 0 or 1", idx);
  if (!t->lens) return fail(AKV_ERR_INVALID, "tier %d: lens is null", idx);
  if (need_slots && !t->slot_base) return fail(AKV_ERR_INVALID, "tier %d: slot_base is null", idx);
  int64_t max_len = 0;
  for (int b = 0; b < B; ++b) {
    if (t->lens[b] < 0) return fail(AKV_ERR_INVALID, "tier %d: lens[%d] = %d < 0", idx, b, t->lens[b]);
    if (t->lens[b] > max_len) max_len = t->lens[b];
    if (need_slots && t->lens[b] > 0) {
      const int64_t ns = ceil_div(t->lens[b], split_tokens);
      if (t->slot_base[b] < 0 || t->slot_base[b] + ns > n_slots)
        return fail(AKV_ERR_INVALID, "tier %d: slots [%d, %lld) of sequence %d outside [0, %lld)", idx,
                    t->slot_base[b], (long long)(t->slot_base[b] + ns), b, (long long)n_slots);
    }
  }
  if (max_len == 0) return AKV_OK;
  if (!t->k || !t->v) return fail(AKV_ERR_INVALID, "tier %d: k or v is null", idx);
  if (!aligned(t->k, 16) || !aligned(t->v, 16)) return fail(AKV_ERR_INVALID, "tier %d: k and v must be 16-byte aligned", idx);
  if (t->stride_seq < 0 || t->stride_head < 0 || t->stride_token < 0)
    return fail(AKV_ERR_INVALID, "tier %d: negative stride", idx);
  if (t->kind == AKV_TIER_BF16) {
    if (t->stride_seq % 8 || t->stride_head % 8 || t->stride_token % 8)
      return fail(AKV_ERR_INVALID, "tier %d: BF16 strides must be multiples of 8 elements", idx);
  }
  if (t->paged) {
    if (!t->page_table) return fail(AKV_ERR_INVALID, "tier %d: paged tier without page_table", idx);
    if (t->n_pages <= 0) return fail(AKV_ERR_INVALID, "tier %d: n_pages must be positive", idx);
    if (t->page_table_stride < ceil_div(max_len, AKV_PAGE_TOKENS))
      return fail(AKV_ERR_INVALID, "tier %d: page_table_stride %lld < %lld pages needed", idx,
                  (long long)t->page_table_stride, (long long)ceil_div(max_len, AKV_PAGE_TOKENS));
  }
  return AKV_OK;
}

akv::TierDev tier_dev(const akv_tier* t) {
  akv::TierDev td;
  td.k = static_cast<const uint8_t*>(t->k);
  td.v = static_cast<const uint8_t*>(t->v);
  td.page_table = t->page_table;
  td.pt_stride = t->page_table_stride;
  td.n_pages = t->n_pages;
  td.s_seq = t->stride_seq;
  td.s_head = t->stride_head;
  td.s_tok = t->stride_token;
  td.paged = t->paged;
  for (int i = 0; i < 4; ++i) td.signs[i] = t->kind == AKV_TIER_CODES4 ? t->rotation_signs[i] : 0u;
  return td;
}

// Fill st for sequences [b0, b0 + n): sequence b owns ceil(len / unit) * mult work
// items; returns the total.
int64_t fill_seq_table(akv::SeqTable& st, int b0, int n, const int32_t* lens, const int32_t* slot_base,
                       int unit, int mult = 1) {
  st.n_seq = n;
  st.b0 = b0;
  int64_t items = 0;
  for (int i = 0; i < n; ++i) {
    st.item_base[i] = (int32_t)items;
    st.len[i] = lens[b0 + i];
    st.slot_base[i] = slot_base ? slot_base[b0 + i] : 0;
    items += ceil_div(lens[b0 + i], unit) * mult;
  }
  st.item_base[n] = (int32_t)items;
  for (int i = n; i < akv::kMaxSeqPerLaunch; ++i) {
    st.len[i] = 0;
    st.slot_base[i] = 0;
    st.item_base[i + 1] = (int32_t)items;
  }
  return items;
}

}  // namespace

namespace akv {

WorkspaceLayout workspace_layout(int B, int Hq, int Hkv, int d, int64_t n_slots) {
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  WorkspaceLayout l;
  l.lse = 0;
  l.o = l.lse + up((size_t)n_slots * Hq * sizeof(float));
  l.total = l.o + up((size_t)n_slots * Hq * d * sizeof(float));
  return l;
}

PFN_cuPointerGetAttribute_v4000 pointer_attribute_fn() {
  static PFN_cuPointerGetAttribute_v4000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuPointerGetAttribute", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuPointerGetAttribute_v4000>(f);
    cudaGetLastError();
  });
  return fn;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    cudaGetLastError();
  });
  return fn;
}



// TMA maps of a BF16 tier.  Logical outer coordinates: 0 token (in the page when paged),
// 1 KV head, 2 sequence (page when paged).  The three outer dims are ordered by byte stride;
// a dim of extent 1 is placed last with a stride past the others.  Boxes are 64 elements x
// 16 tokens with 128-byte swizzle; a box that crosses the extent is zero-filled by TMA.
cudaError_t make_bf16_tensor_maps(AttendParams& p, const akv_tier* t, int B, int Hkv, int d, int64_t max_len) {
  auto encode = tensor_map_encoder();
  if (!encode) return cudaErrorNotSupported;
  uint64_t ext[3] = {t->paged ? (uint64_t)AKV_PAGE_TOKENS : (uint64_t)max_len, (uint64_t)Hkv,
                     t->paged ? (uint64_t)t->n_pages : (uint64_t)B};
  uint64_t str[3] = {(uint64_t)t->stride_token * 2, (uint64_t)t->stride_head * 2, (uint64_t)t->stride_seq * 2};
  uint64_t span = 16;
  for (int i = 0; i < 3; ++i)
    if (ext[i] > 1) span = std::max(span, str[i] * ext[i]);
  for (int i = 0; i < 3; ++i) {
    if (ext[i] > 1 && str[i] == 0) return cudaErrorInvalidValue;  // broadcast strides are not expressible
    if (ext[i] <= 1) str[i] = span + 16 * (uint64_t)(i + 1);
  }
  int order[3] = {0, 1, 2};
  std::sort(order, order + 3, [&](int a, int b) { return str[a] < str[b]; });
  cuuint64_t gdim[4] = {(cuuint64_t)d, ext[order[0]], ext[order[1]], ext[order[2]]};
  cuuint64_t gstr[3] = {str[order[0]], str[order[1]], str[order[2]]};
  cuuint32_t box[4] = {64, 1, 1, 1};
  for (int j = 0; j < 3; ++j)
    if (order[j] == 0) box[j + 1] = AKV_PAGE_TOKENS;
  cuuint32_t estr[4] = {1, 1, 1, 1};
  for (int j = 0; j < 3; ++j) p.tperm[j] = (int8_t)order[j];
  const void* bases[2] = {t->k, t->v};
  CUtensorMap* maps[2] = {&p.tmk, &p.tmv};
  for (int m = 0; m < 2; ++m) {
    CUresult r = encode(maps[m], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(bases[m]), gdim, gstr, box,
                        estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  }
  return cudaSuccess;
}

akv_status set_error(akv_status st, const char* msg) { return fail(st, "%s", msg); }

}  // namespace akv

extern "C" {

int akv_abi_version(void) { return AKV_ABI_VERSION; }

const char* akv_last_error(void) { return g_last_error.c_str(); }

const char* akv_status_string(int status) {
  switch (status) {
    case AKV_OK: return "ok";
    case AKV_ERR_INVALID: return "invalid argument";
    case AKV_ERR_UNSUPPORTED: return "unsupported shape";
    case AKV_ERR_CUDA: return "CUDA error";
    case AKV_ERR_NOT_PINNED: return "host memory is not pinned";
    case AKV_ERR_BUDGET: return "chunk exceeds the staging budget";
    case AKV_ERR_TIMEOUT: return "staging buffer still in use";
    case AKV_ERR_NONFINITE: return "non-finite input";
    case AKV_ERR_RANGE: return "norm out of binary16 range";
    case AKV_ERR_BOUNDS: return "page id out of bounds";
    case AKV_ERR_INTERNAL: return "kernel launch configuration defect";
    default: return "unknown status";
  }
}

akv_status akv_error_word_status(int32_t word) {
  if (word & AKV_EFLAG_INTERNAL) return AKV_ERR_INTERNAL;
  if (word & AKV_EFLAG_TIMEOUT) return AKV_ERR_TIMEOUT;
  if (word & AKV_EFLAG_BOUNDS) return AKV_ERR_BOUNDS;
  if (word & AKV_EFLAG_NONFINITE) return AKV_ERR_NONFINITE;
  if (word & AKV_EFLAG_RANGE) return AKV_ERR_RANGE;
  return AKV_OK;
}

void akv_centroids_f16(uint16_t out[16]) {
  if (out) std::memcpy(out, akv::centroid_table_f16(), 16 * sizeof(uint16_t));
}

akv_status akv_plan_slots(int B, int n_tiers, const int32_t* const* tier_lens, int split_tokens,
                          int32_t* const* tier_slot_base, int32_t* seq_slot_base, int32_t* seq_n_slots,
                          int64_t* n_slots) {
  if (B < 0 || n_tiers < 0) return fail(AKV_ERR_INVALID, "negative B or n_tiers");
  if (split_tokens <= 0) return fail(AKV_ERR_INVALID, "split_tokens must be positive");
  if (!n_slots || (B > 0 && (!seq_slot_base || !seq_n_slots)) || (n_tiers > 0 && (!tier_lens || !tier_slot_base)))
    return fail(AKV_ERR_INVALID, "null output or input array");
  int64_t slot = 0;
  for (int b = 0; b < B; ++b) {
    seq_slot_base[b] = (int32_t)slot;
    for (int i = 0; i < n_tiers; ++i) {
      if (!tier_lens[i] || !tier_slot_base[i]) return fail(AKV_ERR_INVALID, "tier %d arrays are null", i);
      if (tier_lens[i][b] < 0) return fail(AKV_ERR_INVALID, "tier %d: negative length", i);
      tier_slot_base[i][b] = (int32_t)slot;
      slot += ceil_div(tier_lens[i][b], split_tokens);
    }
    seq_n_slots[b] = (int32_t)(slot - seq_slot_base[b]);
    if (slot > INT32_MAX) return fail(AKV_ERR_INVALID, "more than 2^31 slots");
  }
  *n_slots = slot;
  return ok();
}

akv_status akv_append_tokens(const akv_tier* tier, const int32_t* pos, int B, int Hkv, int d, const void* new_k,
                             const void* new_v, int32_t* err_word, akv_stream_t stream) {
  akv::PendingAppend one;
  bool single = false;
  akv_status s = akv::prepare_append(tier, pos, B, Hkv, d, new_k, new_v, err_word, &one, &single);
  if (s != AKV_OK || !one.write) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (single) {
    const cudaError_t e = akv::launch_append(one.p, d, one.n_seq, st);
    return e == cudaSuccess ? ok() : cuda_fail(e, "append launch");
  }
  akv::AppendParams p = one.p;
  for (int b0 = 0; b0 < B; b0 += akv::kMaxSeqPerLaunch) {
    const int n = std::min(akv::kMaxSeqPerLaunch, B - b0);
    p.b0 = b0;
    for (int i = 0; i < n; ++i) p.pos[i] = pos[b0 + i];
    cudaError_t e = akv::launch_append(p, d, n, st);
    if (e != cudaSuccess) return cuda_fail(e, "append launch");
  }
  return ok();
}

}  // extern "C"

namespace akv {

akv_status prepare_append(const akv_tier* tier, const int32_t* pos, int B, int Hkv, int d, const void* new_k,
                          const void* new_v, int32_t* err_word, PendingAppend* out, bool* single) {
  *single = B <= akv::kMaxSeqPerLaunch;
  out->d = d;
  out->n_seq = 0;
  out->write = false;
  if (B < 0 || Hkv <= 0) return fail(AKV_ERR_INVALID, "B must be >= 0 and Hkv > 0");
  if (d != 64 && d != 128) return fail(AKV_ERR_UNSUPPORTED, "head dim %d (supported: 64, 128)", d);
  if (Hkv > 65535) return fail(AKV_ERR_UNSUPPORTED, "Hkv %d too large", Hkv);
  if (!tier) return fail(AKV_ERR_INVALID, "tier is null");
  if (tier->kind != AKV_TIER_BF16) return fail(AKV_ERR_INVALID, "tokens are appended to a BF16 tier");
  if (B == 0) return ok();
  if (!pos) return fail(AKV_ERR_INVALID, "pos is null");
  if (err_word && !aligned(err_word, 4)) return fail(AKV_ERR_INVALID, "err_word must be 4-byte aligned");
  // validate the tier as if it held tokens [0, pos[b]] of every sequence
  std::vector<int32_t> lens(B);
  bool any = false;
  for (int b = 0; b < B; ++b) {
    if (pos[b] == INT32_MAX) return fail(AKV_ERR_INVALID, "pos[%d] too large", b);
    lens[b] = pos[b] < 0 ? 0 : pos[b] + 1;
    any |= pos[b] >= 0;
  }
  if (!any) return ok();  // nothing to write: n_seq stays 0
  if (!new_k || !new_v || !aligned(new_k, 16) || !aligned(new_v, 16))
    return fail(AKV_ERR_INVALID, "new_k and new_v must be 16-byte aligned device pointers");
  akv_tier view = *tier;
  view.lens = lens.data();
  view.slot_base = nullptr;
  akv_status s;
  if ((s = check_tier(&view, 0, B, d, 16, false, 0, AKV_TIER_BF16)) != AKV_OK) return s;
  akv::AppendParams p;
  p.tier = tier_dev(&view);
  p.new_k = static_cast<const uint16_t*>(new_k);
  p.new_v = static_cast<const uint16_t*>(new_v);
  p.err = err_word;
  p.Hkv = Hkv;
  p.b0 = 0;
  out->p = p;
  out->write = true;
  if (*single) {
    for (int i = 0; i < B; ++i) out->p.pos[i] = pos[i];
    out->n_seq = B;
  }
  return ok();
}

}  // namespace akv

extern "C" {


akv_status akv_encode_history(const akv_tier* src, const akv_tier* dst, int B, int Hkv, int d, int32_t* err_word,
                              akv_stream_t stream) {
  if (B < 0 || Hkv <= 0) return fail(AKV_ERR_INVALID, "B must be >= 0 and Hkv > 0");
  if (d != 64 && d != 128) return fail(AKV_ERR_UNSUPPORTED, "head dim %d (supported: 64, 128)", d);
  if (Hkv > 65535) return fail(AKV_ERR_UNSUPPORTED, "Hkv %d too large", Hkv);
  akv_status s;
  if ((s = check_tier(dst, 1, B, d, 16, false, 0, AKV_TIER_CODES4)) != AKV_OK) return s;
  if (!src) return fail(AKV_ERR_INVALID, "source tier is null");
  if (src->kind != AKV_TIER_BF16) return fail(AKV_ERR_INVALID, "source tier must be BF16");
  if (err_word && !aligned(err_word, 4)) return fail(AKV_ERR_INVALID, "err_word must be 4-byte aligned");
  // the source is addressed with the destination's lengths
  akv_tier src_view = *src;
  src_view.lens = dst->lens;
  src_view.slot_base = nullptr;
  if ((s = check_tier(&src_view, 0, B, d, 16, false, 0, AKV_TIER_BF16)) != AKV_OK) return s;
  akv::EncodeParams p;
  p.src = tier_dev(src);
  p.dst = tier_dev(dst);
  p.err = err_word;
  p.Hkv = Hkv;
  std::memcpy(p.bound, akv::centroid_boundaries(), sizeof(p.bound));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  for (int b0 = 0; b0 < B; b0 += akv::kMaxSeqPerLaunch) {
    const int n = std::min(akv::kMaxSeqPerLaunch, B - b0);
    const int64_t items = fill_seq_table(p.seq, b0, n, dst->lens, nullptr, AKV_PAGE_TOKENS);
    if (items == 0) continue;
    if (items > INT32_MAX) return fail(AKV_ERR_UNSUPPORTED, "too many blocks in one launch");
    cudaError_t e = akv::launch_encode(p, d, (int)items, st);
    if (e != cudaSuccess) return cuda_fail(e, "encode launch");
  }
  return ok();
}

}  // extern "C"

namespace {

// One planned attention launch: its parameters, tier kind, (split, KV head) items and the
// tokens of its longest split.
struct PlannedLaunch {
  akv::AttendParams p;
  int kind;
  int items;
  int64_t split_len;
};

// Whether a compact launch and a BF16 launch should share the GPU, and with how many CTAs
// (one per SM) for the compact one.  Estimated durations (fitted to B200 measurements of the
// two kernels, alone and side by side):
//   - a compact split runs on one warp; a 16-token step takes about 0.23 + 0.073 w us when its
//     SM holds w busy warps (they share the SM's issue slots and shared-memory port);
//   - a BF16 split runs on one CTA as 8 chains; a chain step takes about 1.6 us;
//   - a launch that follows another costs about 4 us of ramp and tail.
// The share minimises the larger of the two durations; among equal estimates it is the
// largest, so the compact tier keeps the slack.  It is used only when that beats the two
// launches in a row by 5% or more, which is when one of them would leave SMs or warps idle.
// Returns 0 for "in a row".
int compact_sm_share(int sms, int64_t items_c, int warps_c, int64_t steps_c, int64_t items_x, int64_t chain_steps_x) {
  constexpr double kStepBase = 0.23, kStepPerWarp = 0.073, kBf16ChainStep = 1.6, kLaunch = 4.0, kMargin = 0.95;
  auto t_codes = [&](int ctas) {
    const double busy = std::min<double>((double)warps_c, (double)items_c / ctas);
    return (double)ceil_div(items_c, (int64_t)warps_c * ctas) * steps_c * (kStepBase + kStepPerWarp * busy);
  };
  auto t_bf16 = [&](int ctas) { return (double)ceil_div(items_x, ctas) * chain_steps_x * kBf16ChainStep; };
  const double t_row = t_codes(sms) + t_bf16(sms) + kLaunch;
  int best = 0;
  double best_t = 0.0;
  for (int share = 1; share < sms; ++share) {  // ties go to the larger compact share
    const double t = std::max(t_codes(share), t_bf16(sms - share));
    if (best == 0 || t <= best_t) {
      best_t = t;
      best = share;
    }
  }
  // The estimates are coarse: on the ragged batch (14 waves of compact splits) a share 0.6%
  // below the launches in a row measured 22% slower.  Side by side is kept for the cases it
  // wins clearly (idle SMs or warps otherwise).
  return best_t < kMargin * t_row ? best : 0;
}

// A second stream per device with a fork and a join event.  Created on first use and kept for
// the life of the process; every enqueue sequence that uses it holds side_mutex().
struct SideLane {
  cudaStream_t stream = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};

std::mutex& side_mutex() {
  static std::mutex m;
  return m;
}

cudaError_t side_lane(SideLane*& out) {
  static SideLane lanes[akv::kMaxDevices];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= akv::kMaxDevices) return cudaErrorInvalidDevice;
  SideLane& l = lanes[dev];
  if (!l.stream) {
    SideLane n;
    if ((e = cudaStreamCreateWithFlags(&n.stream, cudaStreamNonBlocking)) != cudaSuccess) return e;
    if ((e = cudaEventCreateWithFlags(&n.fork, cudaEventDisableTiming)) == cudaSuccess &&
        (e = cudaEventCreateWithFlags(&n.join, cudaEventDisableTiming)) == cudaSuccess) {
      l = n;
    } else {
      if (n.fork) cudaEventDestroy(n.fork);
      cudaStreamDestroy(n.stream);
      return e;
    }
  }
  out = &l;
  return cudaSuccess;
}

// The compact launch c on the caller's stream with `share` CTAs, and the BF16 launch x on the
// device's side stream with `rest` CTAs, so the two persistent grids hold disjoint SMs at the
// same time.  The side stream starts after the work enqueued on `st` so far, and `st` resumes
// after both launches; each split's arithmetic is independent of the grid, so the partials
// are the same bits as from two launches in a row.
// Whether `st` belongs to the current device (the side stream's device).  A stream being
// captured into a graph is not asked (the query is not allowed during capture): the call
// must then be made with the stream's device current, as every call on a stream must.
bool stream_on_current_device(cudaStream_t st) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cs) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  if (cs != cudaStreamCaptureStatusNone) return true;
  int cur = 0, dev = 0;
  if (cudaGetDevice(&cur) != cudaSuccess || cudaStreamGetDevice(st, &dev) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return cur == dev;
}

akv_status enqueue_append(const akv::PendingAppend& a, cudaStream_t st) {
  const cudaError_t e = akv::launch_append(a.p, a.d, a.n_seq, st);
  return e == cudaSuccess ? AKV_OK : cuda_fail(e, "append launch");
}

// x (the BF16 tier, after `append` when given) on the side stream, c (the compact tier) on st
akv_status side_by_side(const PlannedLaunch& c, const PlannedLaunch& x, int share, int rest, int d, int G,
                        cudaStream_t st, const akv::PendingAppend* append) {
  std::lock_guard<std::mutex> lock(side_mutex());
  SideLane* lane = nullptr;
  cudaError_t e = side_lane(lane);
  if (e != cudaSuccess) return cuda_fail(e, "side stream");
  if ((e = cudaEventRecord(lane->fork, st)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
  if ((e = cudaStreamWaitEvent(lane->stream, lane->fork, 0)) != cudaSuccess) return cuda_fail(e, "cudaStreamWaitEvent");
  cudaError_t ex = append ? akv::launch_append(append->p, append->d, append->n_seq, lane->stream) : cudaSuccess;
  // after an append on the same stream the launch overlaps it (the kernel waits for the
  // append's writes before its first global read)
  if (ex == cudaSuccess) ex = akv::launch_attend_mma(x.p, d, G, x.kind, x.items, lane->stream, rest, append != nullptr);
  // the join is recorded and waited for even after a failed launch, so `st` never runs ahead of
  // anything the side stream was given
  if ((e = cudaEventRecord(lane->join, lane->stream)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
  const cudaError_t ec =
      ex == cudaSuccess ? akv::launch_attend_mma(c.p, d, G, c.kind, c.items, st, share, true) : cudaSuccess;
  if ((e = cudaStreamWaitEvent(st, lane->join, 0)) != cudaSuccess) return cuda_fail(e, "cudaStreamWaitEvent");
  if (ex != cudaSuccess) return cuda_fail(ex, "attend launch");
  if (ec != cudaSuccess) return cuda_fail(ec, "attend launch");
  return ok();
}

akv_status enqueue_copy_in(const akv::CopyIn& c, cudaStream_t st) {
  const cudaError_t e = c.kernel ? akv::launch_copy_in(c.src, c.dst, c.bytes, st)
                                 : cudaMemcpyAsync(c.dst, c.src, c.bytes, cudaMemcpyHostToDevice, st);
  return e == cudaSuccess ? AKV_OK : cuda_fail(e, "query copy");
}

}  // namespace

namespace akv {

akv_status attend_impl(const void* q, int B, int Hq, int Hkv, int d, float softmax_scale, const akv_tier* tiers,
                       int n_tiers, int split_tokens, float* o_part, float* lse_part, int64_t n_slots, int variant,
                       int32_t* err_word, cudaStream_t st, const CopyIn* copy_in, const PendingAppend* append) {
  if (append && (!append->write || append->n_seq <= 0)) append = nullptr;
  if (B < 0 || n_tiers < 0) return fail(AKV_ERR_INVALID, "negative B or n_tiers");
  if (Hq <= 0 || Hkv <= 0 || Hq % Hkv) return fail(AKV_ERR_INVALID, "Hq must be a positive multiple of Hkv");
  const int G = Hq / Hkv;
  if (!supported_group(G)) return fail(AKV_ERR_UNSUPPORTED, "group size %d (supported: 1, 2, 4, 8)", G);
  if (d != 64 && d != 128) return fail(AKV_ERR_UNSUPPORTED, "head dim %d (supported: 64, 128)", d);
  if (Hkv > 65535) return fail(AKV_ERR_UNSUPPORTED, "Hkv %d too large", Hkv);
  if (split_tokens < 16 || split_tokens > akv::kMaxSplitTokens || split_tokens % 16)
    return fail(AKV_ERR_UNSUPPORTED, "split_tokens %d (a multiple of 16 in [16, 1024])", split_tokens);
  if (!std::isfinite(softmax_scale)) return fail(AKV_ERR_INVALID, "softmax_scale is not finite");
  if (variant != AKV_VARIANT_AUTO && variant != AKV_VARIANT_SIMT && variant != AKV_VARIANT_MMA)
    return fail(AKV_ERR_INVALID, "unknown variant %d", variant);
  if (n_slots < 0) return fail(AKV_ERR_INVALID, "n_slots < 0");
  if (n_tiers > 0 && !tiers) return fail(AKV_ERR_INVALID, "tiers is null");
  if (err_word && !aligned(err_word, 4)) return fail(AKV_ERR_INVALID, "err_word must be 4-byte aligned");
  bool any = false;
  for (int i = 0; i < n_tiers; ++i) {
    akv_status s = check_tier(&tiers[i], i, B, d, split_tokens, true, n_slots, -1);
    if (s != AKV_OK) return s;
    for (int b = 0; b < B; ++b) any |= tiers[i].lens[b] > 0;
  }
  if (!any) return append ? enqueue_append(*append, st) : ok();
  if (!q || !aligned(q, 16)) return fail(AKV_ERR_INVALID, "q must be a 16-byte aligned device pointer");
  if (!o_part || !lse_part) return fail(AKV_ERR_INVALID, "o_part and lse_part must not be null");
  if (!aligned(o_part, 16)) return fail(AKV_ERR_INVALID, "o_part must be 16-byte aligned");
  akv::AttendParams p;
  p.q = static_cast<const uint16_t*>(q);
  p.o_part = o_part;
  p.lse_part = lse_part;
  p.err = err_word;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.split_tokens = split_tokens;
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  std::memcpy(p.centroids, akv::centroid_table_f16(), sizeof(p.centroids));
  // Every launch is checked (and every refusal made) before the first one is enqueued.  The
  // first two launches are kept: that is all the side-by-side case needs, and a call with
  // more launches rebuilds each one's parameters while enqueuing, so no call allocates.
  const bool simt = variant == AKV_VARIANT_SIMT;
  PlannedLaunch two[2];
  int n_launch = 0;
  // pass 0 checks and keeps, pass 1 (more than two launches) enqueues
  for (int pass = 0; pass < 2; ++pass) {
    for (int i = 0; i < n_tiers; ++i) {
      p.tier = tier_dev(&tiers[i]);
      for (int b0 = 0; b0 < B; b0 += akv::kMaxSeqPerLaunch) {
        const int n = std::min(akv::kMaxSeqPerLaunch, B - b0);
        // the CUDA-core kernels take a (split, KV head) grid; the tensor-core kernels a flat
        // list of (split, KV head) items
        const int64_t items =
            fill_seq_table(p.seq, b0, n, tiers[i].lens, tiers[i].slot_base, split_tokens, simt ? 1 : Hkv);
        if (items == 0) continue;
        if (items > INT32_MAX) return fail(AKV_ERR_UNSUPPORTED, "too many splits in one launch");
        int64_t max_len = 0;
        for (int b = b0; b < b0 + n; ++b) max_len = std::max<int64_t>(max_len, tiers[i].lens[b]);
        if (!simt && tiers[i].kind == AKV_TIER_BF16) {
          // global coordinates of the launch's sequences run up to b0 + n
          if (akv::make_bf16_tensor_maps(p, &tiers[i], b0 + n, Hkv, d, max_len) != cudaSuccess)
            return fail(AKV_ERR_UNSUPPORTED, "tier %d: cannot describe its layout to the tensor memory accelerator",
                        i);
        }
        if (pass == 0) {
          if (n_launch < 2) two[n_launch] = PlannedLaunch{p, tiers[i].kind, (int)items, std::min<int64_t>(max_len, split_tokens)};
          ++n_launch;
        } else {
          if (copy_in) {
            const akv_status cs = enqueue_copy_in(*copy_in, st);
            if (cs != AKV_OK) return cs;
            copy_in = nullptr;
          }
          if (append) {
            const akv_status as = enqueue_append(*append, st);
            if (as != AKV_OK) return as;
            append = nullptr;
          }
          // AUTO takes the tensor-core path, which measures faster on both tiers
          cudaError_t e = simt ? akv::launch_attend_simt(p, d, G, tiers[i].kind, (int)items, st)
                               : akv::launch_attend_mma(p, d, G, tiers[i].kind, (int)items, st);
          if (e != cudaSuccess) return cuda_fail(e, "attend launch");
        }
      }
    }
    if (pass == 0 && n_launch <= 2) break;
  }
  if (n_launch > 2) return ok();
  if (copy_in) {  // nothing below refuses
    const akv_status cs = enqueue_copy_in(*copy_in, st);
    if (cs != AKV_OK) return cs;
  }
  const int sms = akv::sm_count();
  if (!simt && n_launch == 2 && two[0].kind != two[1].kind && sms >= 2 && stream_on_current_device(st)) {
    const PlannedLaunch& c = two[0].kind == AKV_TIER_CODES4 ? two[0] : two[1];
    const PlannedLaunch& x = two[0].kind == AKV_TIER_CODES4 ? two[1] : two[0];
    const int share = compact_sm_share(sms, c.items, akv::codes_warps_per_cta(G), ceil_div(c.split_len, 16), x.items,
                                       ceil_div(ceil_div(x.split_len, 16), 8));
    if (share > 0) return side_by_side(c, x, share, sms - share, d, G, st, append);
  }
  if (append) {
    const akv_status as = enqueue_append(*append, st);
    if (as != AKV_OK) return as;
  }
  for (int k = 0; k < n_launch; ++k) {
    const PlannedLaunch& l = two[k];
    cudaError_t e = simt ? akv::launch_attend_simt(l.p, d, G, l.kind, l.items, st)
                         : akv::launch_attend_mma(l.p, d, G, l.kind, l.items, st);
    if (e != cudaSuccess) return cuda_fail(e, "attend launch");
  }
  return ok();
}

}  // namespace akv

extern "C" {

akv_status akv_decode_attend(const void* q, int B, int Hq, int Hkv, int d, float softmax_scale,
                             const akv_tier* tiers, int n_tiers, int split_tokens, float* o_part, float* lse_part,
                             int64_t n_slots, int variant, int32_t* err_word, akv_stream_t stream) {
  return akv::attend_impl(q, B, Hq, Hkv, d, softmax_scale, tiers, n_tiers, split_tokens, o_part, lse_part, n_slots,
                     variant, err_word, reinterpret_cast<cudaStream_t>(stream));
}

akv_status akv_merge_lse(const float* o_part, const float* lse_part, int64_t n_slots, const int32_t* seq_slot_base,
                         const int32_t* seq_n_slots, int B, int Hq, int d, float* o, float* lse,
                         akv_stream_t stream) {
  if (B < 0 || Hq <= 0) return fail(AKV_ERR_INVALID, "B must be >= 0 and Hq > 0");
  if (d != 64 && d != 128) return fail(AKV_ERR_UNSUPPORTED, "head dim %d (supported: 64, 128)", d);
  if (Hq > 65535) return fail(AKV_ERR_UNSUPPORTED, "Hq %d too large", Hq);
  if (B == 0) return ok();
  if (!seq_slot_base || !seq_n_slots) return fail(AKV_ERR_INVALID, "slot arrays are null");
  if (!o || !lse) return fail(AKV_ERR_INVALID, "o and lse must not be null");
  bool any = false;
  for (int b = 0; b < B; ++b) {
    if (seq_n_slots[b] < 0) return fail(AKV_ERR_INVALID, "seq_n_slots[%d] < 0", b);
    if (seq_n_slots[b] > 0 && (seq_slot_base[b] < 0 || (int64_t)seq_slot_base[b] + seq_n_slots[b] > n_slots))
      return fail(AKV_ERR_INVALID, "slots of sequence %d outside [0, %lld)", b, (long long)n_slots);
    any |= seq_n_slots[b] > 0;
  }
  if (any && (!o_part || !lse_part)) return fail(AKV_ERR_INVALID, "o_part and lse_part must not be null");
  if (any && !aligned(o_part, 16)) return fail(AKV_ERR_INVALID, "o_part must be 16-byte aligned");
  akv::MergeParams p;
  p.o_part = o_part;
  p.lse_part = lse_part;
  p.o = o;
  p.lse = lse;
  p.Hq = Hq;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  for (int b0 = 0; b0 < B; b0 += akv::kMaxSeqPerLaunch) {
    const int n = std::min(akv::kMaxSeqPerLaunch, B - b0);
    p.n_seq = n;
    p.b0 = b0;
    for (int i = 0; i < akv::kMaxSeqPerLaunch; ++i) {
      p.slot_base[i] = i < n ? seq_slot_base[b0 + i] : 0;
      p.n_slots[i] = i < n ? seq_n_slots[b0 + i] : 0;
    }
    cudaError_t e = akv::launch_merge(p, d, st);
    if (e != cudaSuccess) return cuda_fail(e, "merge launch");
  }
  return ok();
}

// Plan the standard slot layout for a whole decode step (host vectors).
static akv_status plan_for_decode(int B, const akv_tier* tiers, int n_tiers, int split_tokens,
                                  std::vector<std::vector<int32_t>>& tier_base, std::vector<int32_t>& seq_base,
                                  std::vector<int32_t>& seq_n, int64_t* n_slots) {
  if (B < 0 || n_tiers < 0) return fail(AKV_ERR_INVALID, "negative B or n_tiers");
  if (n_tiers > 0 && !tiers) return fail(AKV_ERR_INVALID, "tiers is null");
  if (split_tokens < 16 || split_tokens > akv::kMaxSplitTokens || split_tokens % 16)
    return fail(AKV_ERR_UNSUPPORTED, "split_tokens %d (a multiple of 16 in [16, 1024])", split_tokens);
  std::vector<const int32_t*> lens(n_tiers);
  std::vector<int32_t*> bases(n_tiers);
  tier_base.assign(n_tiers, std::vector<int32_t>(B > 0 ? B : 1));
  for (int i = 0; i < n_tiers; ++i) {
    if (!tiers[i].lens && B > 0) return fail(AKV_ERR_INVALID, "tier %d: lens is null", i);
    lens[i] = tiers[i].lens;
    bases[i] = tier_base[i].data();
  }
  seq_base.assign(B > 0 ? B : 1, 0);
  seq_n.assign(B > 0 ? B : 1, 0);
  return akv_plan_slots(B, n_tiers, lens.data(), split_tokens, bases.data(), seq_base.data(), seq_n.data(), n_slots);
}

akv_status akv_decode_workspace_size(int B, int Hq, int Hkv, int d, const akv_tier* tiers, int n_tiers,
                                     int split_tokens, size_t* bytes) {
  if (!bytes) return fail(AKV_ERR_INVALID, "bytes is null");
  if (Hq <= 0 || Hkv <= 0 || d <= 0) return fail(AKV_ERR_INVALID, "Hq, Hkv and d must be positive");
  std::vector<std::vector<int32_t>> tb;
  std::vector<int32_t> sb, sn;
  int64_t n_slots = 0;
  akv_status s = plan_for_decode(B, tiers, n_tiers, split_tokens, tb, sb, sn, &n_slots);
  if (s != AKV_OK) return s;
  *bytes = akv::workspace_layout(B, Hq, Hkv, d, n_slots).total;
  return ok();
}

akv_status akv_decode(const void* q, int B, int Hq, int Hkv, int d, float softmax_scale, const akv_tier* tiers,
                      int n_tiers, int split_tokens, void* workspace, size_t workspace_bytes, float* o, float* lse,
                      int variant, int32_t* err_word, akv_stream_t stream) {
  if (Hq <= 0 || Hkv <= 0) return fail(AKV_ERR_INVALID, "Hq and Hkv must be positive");
  std::vector<std::vector<int32_t>> tb;
  std::vector<int32_t> sb, sn;
  int64_t n_slots = 0;
  akv_status s = plan_for_decode(B, tiers, n_tiers, split_tokens, tb, sb, sn, &n_slots);
  if (s != AKV_OK) return s;
  if (B == 0) return ok();
  const akv::WorkspaceLayout lay = akv::workspace_layout(B, Hq, Hkv, d, n_slots);
  if (!workspace || !aligned(workspace, 256)) return fail(AKV_ERR_INVALID, "workspace must be 256-byte aligned");
  if (workspace_bytes < lay.total)
    return fail(AKV_ERR_BUDGET, "workspace of %zu bytes, %zu needed", workspace_bytes, lay.total);
  if (!o || !lse) return fail(AKV_ERR_INVALID, "o and lse must not be null");
  std::vector<akv_tier> planned(tiers, tiers + n_tiers);
  for (int i = 0; i < n_tiers; ++i) planned[i].slot_base = tb[i].data();
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* lse_part = reinterpret_cast<float*>(ws + lay.lse);
  float* o_part = reinterpret_cast<float*>(ws + lay.o);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  s = akv::attend_impl(q, B, Hq, Hkv, d, softmax_scale, planned.data(), n_tiers, split_tokens, o_part, lse_part,
                  n_slots, variant, err_word, st);
  if (s != AKV_OK) return s;
  return akv_merge_lse(o_part, lse_part, n_slots, sb.data(), sn.data(), B, Hq, d, o, lse, stream);
}

}  // extern "C"

namespace {

// Device view of a page-locked host array of `bytes` bytes at p: whether it is page-locked
// host memory the device can address, and the device address of p; `whole` is set when all
// of the array provably lies in that one allocation (the driver reports its range).
struct HostArray {
  bool pinned = false, whole = false;
  void* dev = nullptr;
};

HostArray host_array(const void* p, size_t bytes) {
  HostArray h;
  cudaPointerAttributes a;
  if (!p || cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return h;
  }
  h.pinned = a.type == cudaMemoryTypeHost;
  if (!h.pinned || !a.devicePointer) return h;
  h.dev = a.devicePointer;
  auto get = akv::pointer_attribute_fn();
  CUdeviceptr start = 0;
  size_t size = 0;
  if (get && get(&start, CU_POINTER_ATTRIBUTE_RANGE_START_ADDR, (CUdeviceptr)(uintptr_t)h.dev) == CUDA_SUCCESS &&
      get(&size, CU_POINTER_ATTRIBUTE_RANGE_SIZE, (CUdeviceptr)(uintptr_t)h.dev) == CUDA_SUCCESS) {
    const uintptr_t d0 = (uintptr_t)h.dev;
    h.whole = start != 0 && size != 0 && d0 >= (uintptr_t)start && d0 - (uintptr_t)start <= size &&
              bytes <= size - (d0 - (uintptr_t)start);
  }
  return h;
}

// Byte layout of an akv_decode_host workspace: the query copy, O and LSE (used when the
// outputs go through the copy engine), the LSE partials, the O partials; 256-byte aligned.
struct HostLayout {
  size_t q, o, lse, lse_part, o_part, total;
};

HostLayout host_layout(int B, int Hq, int d, int64_t n_slots) {
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  HostLayout l;
  l.q = 0;
  l.o = up((size_t)B * Hq * d * 2);
  l.lse = l.o + up((size_t)B * Hq * d * sizeof(float));
  l.lse_part = l.lse + up((size_t)B * Hq * sizeof(float));
  l.o_part = l.lse_part + up((size_t)n_slots * Hq * sizeof(float));
  l.total = l.o_part + up((size_t)n_slots * Hq * d * sizeof(float));
  return l;
}

}  // namespace

extern "C" {

akv_status akv_decode_host_workspace_size(int B, int Hq, int Hkv, int d, const akv_tier* tiers, int n_tiers,
                                          int split_tokens, size_t* bytes) {
  if (!bytes) return fail(AKV_ERR_INVALID, "bytes is null");
  if (B < 0 || Hq <= 0 || Hkv <= 0 || d <= 0) return fail(AKV_ERR_INVALID, "B >= 0, Hq, Hkv and d > 0 are required");
  std::vector<std::vector<int32_t>> tb;
  std::vector<int32_t> sb, sn;
  int64_t n_slots = 0;
  akv_status s = plan_for_decode(B, tiers, n_tiers, split_tokens, tb, sb, sn, &n_slots);
  if (s != AKV_OK) return s;
  *bytes = host_layout(B, Hq, d, n_slots).total;
  return ok();
}

akv_status akv_decode_host(const void* q_host, int B, int Hq, int Hkv, int d, float softmax_scale,
                           const akv_tier* tiers, int n_tiers, int split_tokens, void* workspace,
                           size_t workspace_bytes, float* o_host, float* lse_host, int flags, int variant,
                           int32_t* err_word, akv_stream_t stream) {
  if (B < 0 || Hq <= 0 || Hkv <= 0) return fail(AKV_ERR_INVALID, "B >= 0, Hq and Hkv > 0 are required");
  if (flags & ~AKV_HOST_COPY_ENGINE) return fail(AKV_ERR_INVALID, "unknown flags 0x%x", flags);
  if (d != 64 && d != 128) return fail(AKV_ERR_UNSUPPORTED, "head dim %d (supported: 64, 128)", d);
  std::vector<std::vector<int32_t>> tb;
  std::vector<int32_t> sb, sn;
  int64_t n_slots = 0;
  akv_status s = plan_for_decode(B, tiers, n_tiers, split_tokens, tb, sb, sn, &n_slots);
  if (s != AKV_OK) return s;
  if (B == 0) return ok();
  const HostLayout lay = host_layout(B, Hq, d, n_slots);
  if (!workspace || !aligned(workspace, 256)) return fail(AKV_ERR_INVALID, "workspace must be 256-byte aligned");
  if (workspace_bytes < lay.total)
    return fail(AKV_ERR_BUDGET, "workspace of %zu bytes, %zu needed", workspace_bytes, lay.total);
  const size_t q_bytes = (size_t)B * Hq * d * 2, o_bytes = (size_t)B * Hq * d * sizeof(float),
               l_bytes = (size_t)B * Hq * sizeof(float);
  const HostArray hq = host_array(q_host, q_bytes), ho = host_array(o_host, o_bytes), hl = host_array(lse_host, l_bytes);
  if (!hq.pinned || !ho.pinned || !hl.pinned)
    return fail(AKV_ERR_NOT_PINNED, "q_host, o_host and lse_host must be page-locked host memory");
  if (!aligned(q_host, 16) || !aligned(o_host, 4) || !aligned(lse_host, 4))
    return fail(AKV_ERR_INVALID, "q_host must be 16-byte aligned, o_host and lse_host 4-byte aligned");
  // the GPU touches host memory itself only where the driver vouches for the whole array
  const bool kernel_in = !(flags & AKV_HOST_COPY_ENGINE) && hq.whole && aligned(hq.dev, 16);
  const bool kernel_out = !(flags & AKV_HOST_COPY_ENGINE) && ho.whole && hl.whole;
  std::vector<akv_tier> planned(tiers, tiers + n_tiers);
  for (int i = 0; i < n_tiers; ++i) planned[i].slot_base = tb[i].data();
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  void* q_dev = ws + lay.q;
  float* lse_part = reinterpret_cast<float*>(ws + lay.lse_part);
  float* o_part = reinterpret_cast<float*>(ws + lay.o_part);
  const akv::CopyIn copy{kernel_in ? hq.dev : q_host, q_dev, q_bytes, kernel_in};
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  s = akv::attend_impl(q_dev, B, Hq, Hkv, d, softmax_scale, planned.data(), n_tiers, split_tokens, o_part, lse_part,
                       n_slots, variant, err_word, st, &copy);
  if (s != AKV_OK) return s;
  float* o_dst = kernel_out ? static_cast<float*>(ho.dev) : reinterpret_cast<float*>(ws + lay.o);
  float* l_dst = kernel_out ? static_cast<float*>(hl.dev) : reinterpret_cast<float*>(ws + lay.lse);
  s = akv_merge_lse(o_part, lse_part, n_slots, sb.data(), sn.data(), B, Hq, d, o_dst, l_dst, stream);
  if (s != AKV_OK || kernel_out) return s;
  cudaError_t e = cudaMemcpyAsync(o_host, o_dst, o_bytes, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaMemcpyAsync(lse_host, l_dst, l_bytes, cudaMemcpyDeviceToHost, st);
  return e == cudaSuccess ? ok() : cuda_fail(e, "output copy");
}

}  // extern "C"

// ------------------------------------------------------------------------------------
// staging ring
// ------------------------------------------------------------------------------------

struct akv_stager {
  struct Buffer {
    std::vector<cudaEvent_t> pending;  // copies and consumers since the last fill
    cudaEvent_t ready = nullptr;       // the latest fill's copy
  };
  // A write-back into host memory that may still be in flight: a later chunk whose source
  // overlaps [lo, hi) must be copied after it.
  struct HostWrite {
    const uint8_t* lo;
    const uint8_t* hi;
    cudaEvent_t done;
  };
  uint8_t* region = nullptr;
  size_t buf_bytes = 0;
  int n = 0;
  int next = 0;
  std::vector<Buffer> bufs;
  std::vector<HostWrite> host_writes;
  std::vector<cudaEvent_t> free_events;
  std::vector<cudaEvent_t> all_events;
};

namespace {

cudaError_t take_event(akv_stager* st, cudaEvent_t* ev) {
  if (!st->free_events.empty()) {
    *ev = st->free_events.back();
    st->free_events.pop_back();
    return cudaSuccess;
  }
  cudaError_t e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
  if (e == cudaSuccess) st->all_events.push_back(*ev);
  return e;
}

bool is_pinned(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return a.type == cudaMemoryTypeHost;
}

}  // namespace

extern "C" {

akv_status akv_stager_create(void* dev_region, size_t region_bytes, int n_buffers, akv_stager** out) {
  if (!out) return fail(AKV_ERR_INVALID, "out is null");
  *out = nullptr;
  if (!dev_region || region_bytes == 0) return fail(AKV_ERR_INVALID, "empty staging region");
  if (!aligned(dev_region, 256)) return fail(AKV_ERR_INVALID, "staging region must be 256-byte aligned");
  if (n_buffers < 1 || n_buffers > 64) return fail(AKV_ERR_INVALID, "n_buffers %d outside [1, 64]", n_buffers);
  auto* st = new akv_stager;
  st->region = static_cast<uint8_t*>(dev_region);
  st->buf_bytes = (region_bytes / (size_t)n_buffers) / 256 * 256;
  st->n = n_buffers;
  st->bufs.resize(n_buffers);
  if (st->buf_bytes == 0) {
    delete st;
    return fail(AKV_ERR_BUDGET, "region too small for %d buffers", n_buffers);
  }
  *out = st;
  return ok();
}

akv_status akv_stage_chunk(akv_stager* st, const void* pinned_src, size_t bytes, akv_stream_t copy_stream,
                           int timeout_ms, int* buf_index, void** dev_ptr) {
  if (!st || (!pinned_src && bytes) || !buf_index || !dev_ptr) return fail(AKV_ERR_INVALID, "null argument");
  if (bytes > st->buf_bytes)
    return fail(AKV_ERR_BUDGET, "chunk of %zu bytes exceeds the %zu-byte staging buffer", bytes, st->buf_bytes);
  if (bytes && (!is_pinned(pinned_src) || !is_pinned(static_cast<const uint8_t*>(pinned_src) + bytes - 1)))
    return fail(AKV_ERR_NOT_PINNED, "staging source is not page-locked host memory");
  const int idx = st->next;
  akv_stager::Buffer& buf = st->bufs[idx];
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(copy_stream);
  if (timeout_ms >= 0) {
    const auto deadline = std::chrono::steady_clock::now() + std::chrono::milliseconds(timeout_ms);
    for (;;) {
      bool busy = false;
      for (cudaEvent_t ev : buf.pending) {
        cudaError_t q = cudaEventQuery(ev);
        if (q == cudaErrorNotReady) { busy = true; break; }
        if (q != cudaSuccess) return cuda_fail(q, "cudaEventQuery");
      }
      if (!busy) break;
      if (std::chrono::steady_clock::now() >= deadline)
        return fail(AKV_ERR_TIMEOUT, "staging buffer %d still in use after %d ms", idx, timeout_ms);
      std::this_thread::sleep_for(std::chrono::microseconds(50));
    }
  }
  for (cudaEvent_t ev : buf.pending) {
    cudaError_t e = cudaStreamWaitEvent(cs, ev, 0);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamWaitEvent");
  }
  // the copy reads host bytes that an earlier write-back may still be writing: order it
  // after every such write-back; write-backs that have completed are forgotten
  const uint8_t* src_lo = static_cast<const uint8_t*>(pinned_src);
  for (size_t i = 0; i < st->host_writes.size();) {
    akv_stager::HostWrite& w = st->host_writes[i];
    const cudaError_t q = cudaEventQuery(w.done);
    if (q == cudaSuccess) {
      st->free_events.push_back(w.done);
      w = st->host_writes.back();
      st->host_writes.pop_back();
      continue;
    }
    if (q != cudaErrorNotReady) return cuda_fail(q, "cudaEventQuery");
    if (bytes && w.lo < src_lo + bytes && src_lo < w.hi) {
      const cudaError_t e = cudaStreamWaitEvent(cs, w.done, 0);
      if (e != cudaSuccess) return cuda_fail(e, "cudaStreamWaitEvent");
    }
    ++i;
  }
  // a wait binds to the event's latest record at the time of the call, so the events
  // can be recycled now
  for (cudaEvent_t ev : buf.pending) st->free_events.push_back(ev);
  buf.pending.clear();
  buf.ready = nullptr;
  uint8_t* dst = st->region + (size_t)idx * st->buf_bytes;
  cudaError_t e = cudaSuccess;
  if (bytes && (e = cudaMemcpyAsync(dst, pinned_src, bytes, cudaMemcpyHostToDevice, cs)) != cudaSuccess)
    return cuda_fail(e, "cudaMemcpyAsync H2D");
  cudaEvent_t ev;
  if ((e = take_event(st, &ev)) != cudaSuccess) return cuda_fail(e, "cudaEventCreate");
  if ((e = cudaEventRecord(ev, cs)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
  buf.pending.push_back(ev);
  buf.ready = ev;
  st->next = (idx + 1) % st->n;
  *buf_index = idx;
  *dev_ptr = dst;
  return ok();
}

akv_status akv_stager_use(akv_stager* st, int buf_index, akv_stream_t consumer_stream) {
  if (!st || buf_index < 0 || buf_index >= st->n) return fail(AKV_ERR_INVALID, "bad stager or buffer index");
  akv_stager::Buffer& buf = st->bufs[buf_index];
  if (!buf.ready) return fail(AKV_ERR_INVALID, "buffer %d has not been filled", buf_index);
  cudaError_t e = cudaStreamWaitEvent(reinterpret_cast<cudaStream_t>(consumer_stream), buf.ready, 0);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamWaitEvent");
  return ok();
}

akv_status akv_stager_release(akv_stager* st, int buf_index, akv_stream_t consumer_stream) {
  if (!st || buf_index < 0 || buf_index >= st->n) return fail(AKV_ERR_INVALID, "bad stager or buffer index");
  cudaEvent_t ev;
  cudaError_t e = take_event(st, &ev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaEventCreate");
  if ((e = cudaEventRecord(ev, reinterpret_cast<cudaStream_t>(consumer_stream))) != cudaSuccess) {
    st->free_events.push_back(ev);
    return cuda_fail(e, "cudaEventRecord");
  }
  st->bufs[buf_index].pending.push_back(ev);
  return ok();
}

akv_status akv_stage_writeback(akv_stager* st, int buf_index, size_t offset, void* pinned_dst, size_t bytes,
                               akv_stream_t stream) {
  if (!st || buf_index < 0 || buf_index >= st->n || !pinned_dst) return fail(AKV_ERR_INVALID, "bad argument");
  if (bytes == 0) return ok();
  if (offset > st->buf_bytes || bytes > st->buf_bytes - offset)
    return fail(AKV_ERR_BUDGET, "write-back range outside the staging buffer");
  if (!is_pinned(pinned_dst) || !is_pinned(static_cast<uint8_t*>(pinned_dst) + bytes - 1))
    return fail(AKV_ERR_NOT_PINNED, "write-back destination is not page-locked host memory");
  akv_stager::Buffer& buf = st->bufs[buf_index];
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (buf.ready && (e = cudaStreamWaitEvent(s, buf.ready, 0)) != cudaSuccess) return cuda_fail(e, "cudaStreamWaitEvent");
  const uint8_t* src = st->region + (size_t)buf_index * st->buf_bytes + offset;
  if ((e = cudaMemcpyAsync(pinned_dst, src, bytes, cudaMemcpyDeviceToHost, s)) != cudaSuccess)
    return cuda_fail(e, "cudaMemcpyAsync D2H");
  cudaEvent_t done;
  if ((e = take_event(st, &done)) != cudaSuccess) return cuda_fail(e, "cudaEventCreate");
  if ((e = cudaEventRecord(done, s)) != cudaSuccess) {
    st->free_events.push_back(done);
    return cuda_fail(e, "cudaEventRecord");
  }
  const uint8_t* lo = static_cast<const uint8_t*>(pinned_dst);
  st->host_writes.push_back({lo, lo + bytes, done});
  return akv_stager_release(st, buf_index, stream);
}

akv_status akv_stager_destroy(akv_stager* st) {
  if (!st) return ok();
  akv_status result = AKV_OK;
  for (auto& b : st->bufs)
    for (cudaEvent_t ev : b.pending) {
      cudaError_t e = cudaEventSynchronize(ev);
      if (e != cudaSuccess && result == AKV_OK) result = cuda_fail(e, "cudaEventSynchronize");
    }
  for (auto& w : st->host_writes) {
    cudaError_t e = cudaEventSynchronize(w.done);
    if (e != cudaSuccess && result == AKV_OK) result = cuda_fail(e, "cudaEventSynchronize");
  }
  for (cudaEvent_t ev : st->all_events) cudaEventDestroy(ev);
  delete st;
  return result == AKV_OK ? ok() : result;
}

}  // extern "C"

// Whole decode steps behind the C ABI: the staged step of one layer (every chunk of a
// host-resident history staged, attended and released, the new token appended and written
// back, the partials merged) and the live hybrid step whose exact window ages into the
// compact tier.  Each is one library call per step, so the host enqueues a step in
// microseconds instead of issuing the per-chunk and per-tier calls itself.
#include <cstdarg>
#include <cstdio>
#include <vector>

#include "akv_internal.cuh"

namespace {

akv_status refuse(akv_status st, const char* fmt, ...) {
  char buf[384];
  va_list ap;
  va_start(ap, fmt);
  std::vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  return akv::set_error(st, buf);
}

int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

}  // namespace

// ------------------------------------------------------------------------------------
// staged step of one layer
// ------------------------------------------------------------------------------------

extern "C" akv_status akv_staged_decode(akv_stager* stager, const akv_staged_history* hist, const void* q, int Hq,
                                        int Hkv, int d, float softmax_scale, int split_tokens, const void* new_row,
                                        const akv_tier* window, float* o_part, float* lse_part, int64_t n_slots,
                                        float* o, float* lse, int variant, int32_t* err_word,
                                        akv_stream_t copy_stream, akv_stream_t compute_stream) {
  if (!stager || !hist || !q || !o_part || !lse_part || !o || !lse)
    return refuse(AKV_ERR_INVALID, "akv_staged_decode: null argument");
  if (d != 64 && d != 128) return refuse(AKV_ERR_UNSUPPORTED, "head dim %d (supported: 64, 128)", d);
  if (Hkv <= 0 || Hq <= 0 || Hq % Hkv) return refuse(AKV_ERR_INVALID, "Hq must be a positive multiple of Hkv");
  if (split_tokens < 16 || split_tokens > akv::kMaxSplitTokens || split_tokens % 16)
    return refuse(AKV_ERR_UNSUPPORTED, "split_tokens must be a multiple of 16 in [16, 1024]");
  const bool codes = hist->kind == AKV_TIER_CODES4;
  if (hist->kind != AKV_TIER_BF16 && !codes) return refuse(AKV_ERR_INVALID, "unknown history kind %d", hist->kind);
  if (hist->n_tokens < 0) return refuse(AKV_ERR_INVALID, "negative history length");
  if (hist->n_tokens > 0 && !hist->host) return refuse(AKV_ERR_INVALID, "history without host rows");
  const int64_t chunk = hist->chunk_tokens;
  if (chunk <= 0 || chunk % split_tokens)
    return refuse(AKV_ERR_INVALID, "chunk_tokens must be a positive multiple of split_tokens");
  if (codes && new_row) return refuse(AKV_ERR_INVALID, "a compact history takes no appended row");
  if (window && (window->kind != AKV_TIER_BF16 || !window->lens || window->lens[0] < 0))
    return refuse(AKV_ERR_INVALID, "the window must be a BF16 tier with lens[0] >= 0");
  const int64_t bb = AKV_CODES4_BLOCK_BYTES(d);
  // bytes of one history row: a BF16 token [K | V][Hkv][d], or a 16-token code block row
  const int64_t row_bytes = codes ? 2 * (int64_t)Hkv * bb : 2 * (int64_t)Hkv * d * 2;
  const int64_t n_hist = hist->n_tokens + (new_row ? 1 : 0);
  const int64_t hist_splits = cdiv(n_hist, split_tokens);
  const int64_t win_len = window ? window->lens[0] : 0;
  const int64_t total_splits = hist_splits + cdiv(win_len, split_tokens);
  if (total_splits > n_slots) return refuse(AKV_ERR_BUDGET, "%lld slots needed, %lld given", (long long)total_splits,
                                            (long long)n_slots);
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(compute_stream);
  const uint8_t* host = static_cast<const uint8_t*>(hist->host);
  const int64_t per_chunk = chunk / split_tokens;
  const int64_t pos = hist->n_tokens;  // the appended token's position
  for (int64_t c = 0; c * chunk < n_hist; ++c) {
    const int64_t tok0 = c * chunk;
    const int64_t ntc = n_hist - tok0 < chunk ? n_hist - tok0 : chunk;
    int64_t src_off, bytes;
    if (codes) {
      src_off = (tok0 / 16) * row_bytes;
      bytes = cdiv(ntc, 16) * row_bytes;
    } else {  // the appended row is not in the host copy yet
      const int64_t have = hist->n_tokens - tok0 < ntc ? hist->n_tokens - tok0 : ntc;
      src_off = tok0 * row_bytes;
      bytes = have > 0 ? have * row_bytes : 0;
    }
    int buf = -1;
    void* dev = nullptr;
    akv_status s = akv_stage_chunk(stager, host + src_off, (size_t)bytes, copy_stream, -1, &buf, &dev);
    if (s != AKV_OK) return s;
    if ((s = akv_stager_use(stager, buf, compute_stream)) != AKV_OK) return s;
    uint8_t* base = static_cast<uint8_t*>(dev);
    const bool appends = new_row && tok0 <= pos && pos < tok0 + chunk;
    if (appends) {
      const cudaError_t e = cudaMemcpyAsync(base + (pos - tok0) * row_bytes, new_row, (size_t)row_bytes,
                                            cudaMemcpyDeviceToDevice, cs);
      if (e != cudaSuccess) return refuse(AKV_ERR_CUDA, "append copy: %s", cudaGetErrorString(e));
    }
    const int32_t lens[1] = {(int32_t)ntc};
    const int32_t slot[1] = {(int32_t)(c * per_chunk)};
    akv_tier t = {};
    t.kind = hist->kind;
    t.k = base;
    t.lens = lens;
    t.slot_base = slot;
    t.stride_seq = 0;
    if (codes) {
      t.v = base + Hkv * bb;
      t.stride_head = 1;
      t.stride_token = 2 * Hkv;
      for (int i = 0; i < 4; ++i) t.rotation_signs[i] = hist->rotation_signs[i];
    } else {
      t.v = base + (int64_t)Hkv * d * 2;
      t.stride_head = d;
      t.stride_token = 2 * (int64_t)Hkv * d;
    }
    s = akv_decode_attend(q, 1, Hq, Hkv, d, softmax_scale, &t, 1, split_tokens, o_part, lse_part, n_slots, variant,
                          err_word, compute_stream);
    if (s != AKV_OK) return s;
    s = appends ? akv_stage_writeback(stager, buf, (size_t)((pos - tok0) * row_bytes),
                                      const_cast<uint8_t*>(host) + pos * row_bytes, (size_t)row_bytes, compute_stream)
                : akv_stager_release(stager, buf, compute_stream);
    if (s != AKV_OK) return s;
  }
  if (win_len > 0) {
    akv_tier w = *window;
    const int32_t slot[1] = {(int32_t)hist_splits};
    w.slot_base = slot;
    const akv_status s = akv_decode_attend(q, 1, Hq, Hkv, d, softmax_scale, &w, 1, split_tokens, o_part, lse_part,
                                           n_slots, variant, err_word, compute_stream);
    if (s != AKV_OK) return s;
  }
  const int32_t seq_base[1] = {0}, seq_n[1] = {(int32_t)total_splits};
  return akv_merge_lse(o_part, lse_part, n_slots, seq_base, seq_n, 1, Hq, d, o, lse, compute_stream);
}

// ------------------------------------------------------------------------------------
// window aging
// ------------------------------------------------------------------------------------

namespace akv {
namespace {

constexpr int kAgeMax = kMaxSeqPerLaunch;

struct AgeParams {
  int32_t* compact_table;  // device [B][compact_stride]
  int64_t compact_stride;
  int32_t* window_table;   // device [B][R]
  int32_t* lists;          // device [2 n]: (source window page, destination code page) per aging sequence
  int32_t R;
  int32_t n;
  int32_t list0;           // first list entry written by this launch
  int32_t b[kAgeMax];
  int32_t slot[kAgeMax];   // logical code page the new page takes
  int32_t page[kAgeMax];   // the code page
  int32_t src[kAgeMax];    // the window pool page leaving the window
  int32_t head[kAgeMax];   // ring slot of the window's first page after aging
};

// One block per aging sequence: enter the code page, rotate the window's page-table row and
// write the encode's page list.
__global__ void age_tables_kernel(const __grid_constant__ AgeParams p) {
  const int i = blockIdx.x;
  const int b = p.b[i];
  if (threadIdx.x == 0) {
    p.compact_table[(int64_t)b * p.compact_stride + p.slot[i]] = p.page[i];
    p.lists[2 * (p.list0 + i)] = p.src[i];
    p.lists[2 * (p.list0 + i) + 1] = p.page[i];
  }
  for (int j = threadIdx.x; j < p.R; j += blockDim.x) p.window_table[(int64_t)b * p.R + j] = b * p.R + (p.head[i] + j) % p.R;
}

}  // namespace
}  // namespace akv

struct akv_aging {
  akv_aging_desc desc;
  akv_tier window, compact;                 // copies; lens and slot bases point at the vectors below
  std::vector<int32_t> c, win, head;        // compact tokens, window tokens, ring slot of the first page
  std::vector<std::vector<int32_t>> pages;  // each sequence's code pages, in the order it takes them
  std::vector<int32_t> pos, cbase, wbase, seq_base, seq_n;
  std::vector<int32_t> ones16;
  int64_t n_slots = 0;
  int64_t steps = 0, aged = 0;
};

extern "C" akv_status akv_aging_create(const akv_aging_desc* dsc, akv_aging** out) {
  if (!out) return refuse(AKV_ERR_INVALID, "out is null");
  *out = nullptr;
  if (!dsc) return refuse(AKV_ERR_INVALID, "desc is null");
  const akv_aging_desc& a = *dsc;
  if (a.B <= 0 || a.Hkv <= 0 || a.Hq <= 0 || a.Hq % a.Hkv) return refuse(AKV_ERR_INVALID, "bad B, Hq or Hkv");
  if (a.d != 64 && a.d != 128) return refuse(AKV_ERR_UNSUPPORTED, "head dim %d (supported: 64, 128)", a.d);
  if (a.window_tokens <= 0 || a.window_tokens % 16) return refuse(AKV_ERR_INVALID, "window_tokens: positive multiple of 16");
  const int R = a.ring_pages;
  if (R < a.window_tokens / 16 + 2) return refuse(AKV_ERR_INVALID, "ring_pages must be at least window_tokens / 16 + 2");
  if (a.window.kind != AKV_TIER_BF16 || !a.window.paged || !a.window.page_table || a.window.page_table_stride != R)
    return refuse(AKV_ERR_INVALID, "window: a paged BF16 tier whose page-table rows hold ring_pages entries");
  if ((int64_t)a.B * R > a.window.n_pages) return refuse(AKV_ERR_INVALID, "window pool smaller than B * ring_pages");
  if (a.compact.kind != AKV_TIER_CODES4 || !a.compact.paged || !a.compact.page_table)
    return refuse(AKV_ERR_INVALID, "compact: a paged CODES4 tier");
  if (!a.compact_len || !a.window_len || !a.ring_head || !a.page_lists || !a.page_list_len || !a.lists_dev ||
      !a.o_part || !a.lse_part)
    return refuse(AKV_ERR_INVALID, "null array in desc");
  auto* g = new akv_aging;
  g->desc = a;
  g->c.assign(a.compact_len, a.compact_len + a.B);
  g->win.assign(a.window_len, a.window_len + a.B);
  g->head.assign(a.ring_head, a.ring_head + a.B);
  g->pages.resize(a.B);
  for (int b = 0; b < a.B; ++b) {
    if (g->c[b] < 0 || g->c[b] % 16 || g->win[b] < a.window_tokens || g->win[b] >= a.window_tokens + 16 ||
        g->head[b] < 0 || g->head[b] >= R || a.page_list_len[b] < g->c[b] / 16 ||
        a.page_list_len[b] > a.compact.page_table_stride || (a.page_list_len[b] && !a.page_lists[b])) {
      delete g;
      return refuse(AKV_ERR_INVALID, "sequence %d: lengths, ring head or page list out of range", b);
    }
    g->pages[b].assign(a.page_lists[b], a.page_lists[b] + a.page_list_len[b]);
  }
  g->window = a.window;
  g->compact = a.compact;
  g->pos.resize(a.B);
  g->cbase.resize(a.B);
  g->wbase.resize(a.B);
  g->seq_base.resize(a.B);
  g->seq_n.resize(a.B);
  g->ones16.assign(a.B, 16);
  *out = g;
  return AKV_OK;
}

extern "C" akv_status akv_aging_step(akv_aging* g, const void* q, const void* k_new, const void* v_new, float* o,
                                     float* lse, int variant, int32_t* err_word, akv_stream_t stream) {
  if (!g || !q || !k_new || !v_new || !o || !lse) return refuse(AKV_ERR_INVALID, "akv_aging_step: null argument");
  const akv_aging_desc& a = g->desc;
  const int B = a.B, R = a.ring_pages;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // every sequence that would run out of code pages is refused before anything is enqueued
  for (int b = 0; b < B; ++b)
    if (g->win[b] + 1 >= a.window_tokens + 16 && g->c[b] / 16 >= (int32_t)g->pages[b].size())
      return refuse(AKV_ERR_BUDGET, "sequence %d has no code page left to age into", b);
  // 1. the new token goes to position win[b] of the window.  A step that ages a page
  // enqueues the append first (the aging rewrites the window's page table); otherwise the
  // append is handed to the attention call, which runs it just before the window's launch
  // (beside the compact tier when the two tiers share the GPU).
  for (int b = 0; b < B; ++b) g->pos[b] = g->win[b];
  bool ages = false;
  for (int b = 0; b < B; ++b) ages |= g->win[b] + 1 >= a.window_tokens + 16;
  akv_tier wt = g->window;
  wt.lens = g->win.data();
  akv::PendingAppend app;
  bool single = false;
  akv_status st = akv::prepare_append(&wt, g->pos.data(), B, a.Hkv, a.d, k_new, v_new, err_word, &app, &single);
  if (st != AKV_OK) return st;
  const bool deferred = single && !ages;
  if (!deferred) {
    st = akv_append_tokens(&wt, g->pos.data(), B, a.Hkv, a.d, k_new, v_new, err_word, stream);
    if (st != AKV_OK) return st;
  }
  // 2. a window of W + 16 tokens hands its oldest page to the compact tier
  std::vector<int> aging;
  for (int b = 0; b < B; ++b) {
    ++g->win[b];
    if (g->win[b] >= a.window_tokens + 16) aging.push_back(b);
  }
  if (!aging.empty()) {
    const int n = (int)aging.size();
    for (int i0 = 0; i0 < n; i0 += akv::kAgeMax) {
      akv::AgeParams p = {};
      p.compact_table = const_cast<int32_t*>(a.compact.page_table);
      p.compact_stride = a.compact.page_table_stride;
      p.window_table = const_cast<int32_t*>(a.window.page_table);
      p.lists = a.lists_dev;
      p.R = R;
      p.n = n - i0 < akv::kAgeMax ? n - i0 : akv::kAgeMax;
      p.list0 = i0;
      for (int i = 0; i < p.n; ++i) {
        const int b = aging[i0 + i];
        p.b[i] = b;
        p.slot[i] = g->c[b] / 16;
        p.page[i] = g->pages[b][g->c[b] / 16];
        p.src[i] = b * R + g->head[b];
        g->c[b] += 16;
        g->head[b] = (g->head[b] + 1) % R;
        g->win[b] -= 16;
        p.head[i] = g->head[b];
      }
      akv::age_tables_kernel<<<p.n, 32, 0, s>>>(p);
      const cudaError_t e = cudaGetLastError();
      if (e != cudaSuccess) return refuse(AKV_ERR_CUDA, "age_tables_kernel: %s", cudaGetErrorString(e));
    }
    // the leaving pages: column 0 of the lists addresses the window pages, column 1 the code pages
    akv_tier src = g->window, dst = g->compact;
    src.lens = dst.lens = g->ones16.data();
    src.page_table = dst.page_table = a.lists_dev;
    dst.page_table = a.lists_dev + 1;
    src.page_table_stride = dst.page_table_stride = 2;
    st = akv_encode_history(&src, &dst, n, a.Hkv, a.d, err_word, stream);
    if (st != AKV_OK) return st;
    g->aged += n;
  }
  // 3. both tiers into their planned slots, then the merge
  const int32_t* lens[2] = {g->c.data(), g->win.data()};
  int32_t* bases[2] = {g->cbase.data(), g->wbase.data()};
  st = akv_plan_slots(B, 2, lens, a.split_tokens, bases, g->seq_base.data(), g->seq_n.data(), &g->n_slots);
  if (st != AKV_OK) return st;
  if (g->n_slots > a.n_slots) return refuse(AKV_ERR_BUDGET, "%lld slots needed, %lld given", (long long)g->n_slots,
                                            (long long)a.n_slots);
  akv_tier tiers[2] = {g->compact, g->window};
  tiers[0].lens = g->c.data();
  tiers[0].slot_base = g->cbase.data();
  tiers[1].lens = g->win.data();
  tiers[1].slot_base = g->wbase.data();
  st = akv::attend_impl(q, B, a.Hq, a.Hkv, a.d, a.softmax_scale, tiers, 2, a.split_tokens, a.o_part, a.lse_part,
                        a.n_slots, variant, err_word, s, nullptr, deferred ? &app : nullptr);
  if (st != AKV_OK) {
    // the window now counts the new token: write it even though the step fails (writing it
    // twice stores the same row)
    if (deferred) akv_append_tokens(&wt, g->pos.data(), B, a.Hkv, a.d, k_new, v_new, err_word, stream);
    return st;
  }
  st = akv_merge_lse(a.o_part, a.lse_part, a.n_slots, g->seq_base.data(), g->seq_n.data(), B, a.Hq, a.d, o, lse,
                     stream);
  if (st != AKV_OK) return st;
  ++g->steps;
  return AKV_OK;
}

extern "C" akv_status akv_aging_state(const akv_aging* g, int32_t* compact_len, int32_t* window_len,
                                      int32_t* ring_head, int64_t* aged_pages) {
  if (!g) return refuse(AKV_ERR_INVALID, "akv_aging_state: null context");
  const int B = g->desc.B;
  for (int b = 0; b < B; ++b) {
    if (compact_len) compact_len[b] = g->c[b];
    if (window_len) window_len[b] = g->win[b];
    if (ring_head) ring_head[b] = g->head[b];
  }
  if (aged_pages) *aged_pages = g->aged;
  return AKV_OK;
}

extern "C" akv_status akv_aging_destroy(akv_aging* g) {
  delete g;
  return AKV_OK;
}

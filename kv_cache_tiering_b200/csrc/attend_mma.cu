// Split-KV GQA decode attention on the tensor cores (mma.sync m16n8k16, float32
// accumulate), contracting across the GQA query group.
//
// Work decomposition.  A work item is one split of one sequence for one KV head and its
// G query heads.  Every split is computed as NW chains: chain w owns the 16-token steps
// w, w + NW, w + 2 NW, ... and keeps its own online-softmax state; the chain states are
// merged in chain order at the end of the split.  This decomposition is fixed, so the
// value written for a split never depends on how many items a call holds or where its
// tokens live (a staged run equals the resident run bit for bit).
//
// Launch.  The grid is persistent: at most one CTA per SM, each owning a contiguous,
// equal-length range of items (item order is sequence, then KV head, then split, so
// consecutive items share their query).  Exact tier: NW = 8 chains per split, warp w runs
// chain w of every item of the CTA back to back.  Compact tier: one chain per split, each
// warp owns its own item range.  Every warp streams its steps through a private ring of
// NST shared-memory stages that keeps prefetching across item boundaries.  BF16 stages are
// TMA tiles (cp.async.bulk.tensor, 128-byte swizzle) issued by one lane, each completing on
// its own mbarrier; every mbarrier wait is bounded: a wait that runs out sets
// AKV_EFLAG_TIMEOUT and the warp stops computing, drains its copies (again bounded) and
// leaves.  Compact stages are the key and value blocks as stored, copied by all 32 lanes in
// 16-byte cp.async.cg chunks, one commit group per step.
//
// Exact BF16 tier, per step (16 tokens):
//   S^T (16 rows x 16 tokens) = q . K^T     A = q rows (heads), B = K rows via ldmatrix
//   O^T (d x 8 cols)         += V^T . P^T   A = V via ldmatrix.trans, B = P from the S^T
//                                           accumulator registers
// The weights P carry a BF16 high part and a BF16 residual: for G <= 4 the residual of
// head h rides in PV column 4 + h of the same MMA, for G = 8 in a second MMA.
// The TMA swizzle puts 16-byte chunk j of tile row r at chunk j ^ (r & 7) of its 128-byte
// line, so the ldmatrix row gathers are conflict-free.
//
// Compact tier, per step: the same contractions in the rotated basis ("QuantForge V2
// Walkthrough", section 1: rotate the query instead of the keys) with FP16 operands.
//   S (16 tokens x 8 cols) = K_hat . Q^T   A = dequantised keys, B = the rotated query
//   O^T (d x 8 cols)      += V_hat^T . P^T A = dequantised values, B = the weights
// Code bytes become (c[lo], c[hi]) half pairs through a per-lane replicated table in
// shared memory, each lookup one A-fragment entry; value code nibbles of two tokens share
// a byte, so one entry is a (token, token) pair at one dimension.  The rotated query H q is
// an FP16 high part and an FP16 residual (for G <= 4 head h's are columns h and h + 4, for
// G = 8 a second product), so scores keep ~22 significant bits; the weights are split the
// same way.  The key scale multiplies the scores, the value scale the weights, and the
// output is rotated back with a Walsh-Hadamard transform over shuffles.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "akv_internal.cuh"

namespace akv {
namespace {

constexpr float kLn2 = 0.693147180559945309f;
constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
// ---- mbarriers, TMA and bulk copies
constexpr uint32_t kWaitLimit = 1u << 22;  // try_wait rounds before a wait gives up

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(bar), "r"(bytes) : "memory");
}
// Bounded wait for phase `parity` of an mbarrier; false when the wait ran out.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  for (uint32_t i = 0; i < kWaitLimit; ++i) {
    uint32_t done;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    if (done) return true;
  }
  return false;
}
// L2 policy of the K/V streams: every history byte is read once per launch, so its lines
// are the first to go and the queries, page tables and partial outputs (read again by the
// merge) stay in L2.  Worth 3-4% on the BF16 tier and about 2% on the compact tier.
__device__ __forceinline__ uint64_t l2_evict_first() {
  uint64_t pol;
  asm("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;\n" : "=l"(pol));  // pure: may be re-issued
  return pol;
}
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, int c0, int c1, int c2, int c3,
                                            uint32_t bar, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4, %5}], [%6], %7;\n" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar), "l"(pol)
      : "memory");
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint64_t pol) {
  asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "l"(pol));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
// The MMAs are plain asm: their results depend only on their operands, so the compiler may
// interleave them with independent work.
__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_f16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// Shared-memory loads on 32-bit shared-window addresses, with an immediate offset.  Ring
// stages are read with volatile asm, which keeps each read after the cp.async wait that
// publishes the stage; table reads are plain, the table being constant once built.
template <int OFF = 0>
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1+%2];\n" : "=r"(v) : "r"(a), "n"(OFF));
  return v;
}
template <int OFF = 0>
__device__ __forceinline__ uint2 lds64(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.b32 {%0, %1}, [%2+%3];\n" : "=r"(v.x), "=r"(v.y) : "r"(a), "n"(OFF));
  return v;
}
template <int OFF = 0>
__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4+%5];\n"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(a), "n"(OFF));
  return v;
}
template <int OFF = 0>
__device__ __forceinline__ float lds_half(uint32_t a) {  // one binary16 from a ring stage, as float
  unsigned short v;
  asm volatile("ld.shared.u16 %0, [%1+%2];\n" : "=h"(v) : "r"(a), "n"(OFF));
  return __half2float(__ushort_as_half(v));
}
// 8 x 8 transpose of 16-bit elements across the warp: lane (r, c) holding row r, columns
// 2c, 2c + 1 receives row r of the transpose (column r, rows 2c, 2c + 1 of the input).
__device__ __forceinline__ uint32_t transpose8x8(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
  return y;
}
__device__ __forceinline__ uint32_t lds32_const(uint32_t a) {
  uint32_t v;
  asm("ld.shared.b32 %0, [%1];\n" : "=r"(v) : "r"(a));
  return v;
}
// 2^x on the special-function unit (ex2.approx: relative error about 2^-22, -inf -> +0,
// subnormal results flushed to zero).
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float2 unpack_f16(uint32_t w) {
  return __half22float2(*reinterpret_cast<const __half2*>(&w));
}
// named barrier of one warp group (ids 1.. ; 0 is __syncthreads)
template <int NW>
__device__ __forceinline__ void group_sync(int gi) {
  asm volatile("bar.sync %0, %1;\n" ::"r"(gi + 1), "n"(NW * 32) : "memory");
}

// ------------------------------------------------------------------------------------
// items
// ------------------------------------------------------------------------------------
struct Item {
  int bl;     // sequence within the launch
  int b;      // global sequence
  int kvh;
  int t0;     // first token of the split (tier-relative)
  int n;      // tokens in the split
  int slot;
  int pair;   // b * Hkv + kvh: items with the same pair share their query
};

// The launch's sequence table, copied into shared memory once per CTA: finding an item's
// sequence is a binary search, and its dependent reads cost less from shared memory than
// from the parameter bank (2% on the compact tier at batch 4).
struct SeqSmem {
  int32_t item_base[kMaxSeqPerLaunch + 1];
  int32_t len[kMaxSeqPerLaunch];
  int32_t slot_base[kMaxSeqPerLaunch];
};
__device__ __forceinline__ void fill_seq_smem(const AttendParams& p, SeqSmem* ss) {
  const int n = p.seq.n_seq;
  for (int i = threadIdx.x; i <= n; i += blockDim.x) {
    ss->item_base[i] = p.seq.item_base[i];
    if (i < n) {
      ss->len[i] = p.seq.len[i];
      ss->slot_base[i] = p.seq.slot_base[i];
    }
  }
}

// Item order: sequence, KV head, split.  seq.item_base counts splits * Hkv per sequence.
// ss: the shared-memory copy of the sequence table, or null to read the parameters.
__device__ __forceinline__ Item item_at(const AttendParams& p, int item, const SeqSmem* ss) {
  int bl = 0;
  if (ss) {
    int hi = p.seq.n_seq - 1;
    while (bl < hi) {
      const int mid = (bl + hi + 1) >> 1;
      if (ss->item_base[mid] <= item) bl = mid; else hi = mid - 1;
    }
  } else {
    bl = find_seq(p.seq, item);
  }
  const int r = item - (ss ? ss->item_base[bl] : p.seq.item_base[bl]);
  const int len = ss ? ss->len[bl] : p.seq.len[bl];
  const int ns = (len + p.split_tokens - 1) / p.split_tokens;
  Item it;
  it.kvh = r / ns;
  const int split = r - it.kvh * ns;
  it.bl = bl;
  it.b = p.seq.b0 + bl;
  it.t0 = split * p.split_tokens;
  it.n = min(p.split_tokens, len - it.t0);
  it.slot = (ss ? ss->slot_base[bl] : p.seq.slot_base[bl]) + split;
  it.pair = it.b * p.Hkv + it.kvh;
  return it;
}

// Contiguous item range [lo, hi) of this CTA; group gi takes lo + gi, lo + gi + NG, ...
__device__ __forceinline__ void cta_range(int total, int& lo, int& hi) {
  const int q = total / (int)gridDim.x, r = total % (int)gridDim.x, c = blockIdx.x;
  lo = c * q + min(c, r);
  hi = lo + q + (c < r ? 1 : 0);
}

// Chain-ordered cursor over (item, step) pairs of one warp: steps w, w + NW, ... of each
// item of the group, items in group order.
struct Cursor {
  int item;   // absolute item index, >= hi when exhausted
  int step;
  Item info;
};

template <int NG>
__device__ __forceinline__ void cursor_settle(const AttendParams& p, Cursor& c, int hi, int w, const SeqSmem* ss) {
  // move forward until the cursor sits on a step that exists
  while (c.item < hi && 16 * c.step >= c.info.n) {
    c.item += NG;
    c.step = w;
    if (c.item < hi) c.info = item_at(p, c.item, ss);
  }
}

template <int NW, int NG>
__device__ __forceinline__ void cursor_next(const AttendParams& p, Cursor& c, int hi, int w, const SeqSmem* ss) {
  c.step += NW;
  cursor_settle<NG>(p, c, hi, w, ss);
}

// ------------------------------------------------------------------------------------
// online softmax of one step.  sc[j][e] (e < 2): base-2 scores of head g for tokens
// 8j + 2tq + e, masked with -inf.  The running reference m_run of a head sits kSlack above
// a maximum already seen, so the weights 2^(s - m_run) stay at most 1; only a score above
// m_run (in practice a chain's first steps) costs the cross-lane maximum, and then the
// function returns true with the rescale factors of the accumulator columns 2tq, 2tq + 1
// (column c holds head c for G = 8 and head c % 4 for G <= 4).  LSE = m_run + log2 l_run
// holds for any reference.  Leaves the weights in sc[j][e].
// ------------------------------------------------------------------------------------
template <int G, int N>
__device__ __forceinline__ bool online_softmax(float (&sc)[2][N], float& m_run, float& l_run, float& a_even,
                                               float& a_odd) {
  constexpr float kSlack = 8.f;
  const int lane = threadIdx.x & 31, tq = lane & 3;
  float mx = fmaxf(fmaxf(sc[0][0], sc[0][1]), fmaxf(sc[1][0], sc[1][1]));
  bool rescale = false;
  if (__any_sync(kFull, mx > m_run)) {
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
    const float m_new = fmaxf(m_run, mx + kSlack);
    const float alpha = fast_exp2(m_run - m_new);  // 0 while m_run = -inf
    l_run *= alpha;
    m_run = m_new;
    constexpr int HM = G <= 4 ? 3 : 7;
    a_even = __shfl_sync(kFull, alpha, ((2 * tq) & HM) * 4);
    a_odd = __shfl_sync(kFull, alpha, ((2 * tq + 1) & HM) * 4);
    rescale = true;
  }
  float s = 0.f;
#pragma unroll
  for (int j = 0; j < 2; ++j)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      sc[j][e] = fast_exp2(sc[j][e] - m_run);
      s += sc[j][e];
    }
  l_run += s;
  return rescale;
}

// P^T B fragments from the weights w[j][e] (head g, tokens 8j + 2tq + e): high part and
// residual in the MMA type.  G <= 4: one fragment, columns 0..3 high parts and 4..7 the
// residuals of heads 0..3 (lanes of group g >= 4 take lane ^ 16's residual).
template <int G, bool kBF16>
__device__ __forceinline__ void p_fragments(const float (&w)[2][2], uint32_t (&b_hi)[2], uint32_t (&b_lo)[2]) {
  const int g = (threadIdx.x & 31) >> 2;
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    uint32_t hi, lo;
    if constexpr (kBF16) {
      hi = pack_bf16(w[j][0], w[j][1]);
      lo = pack_bf16(w[j][0] - __uint_as_float(hi << 16), w[j][1] - __uint_as_float(hi & 0xffff0000u));
    } else {
      hi = pack_f16(w[j][0], w[j][1]);
      const float2 h = unpack_f16(hi);
      lo = pack_f16(w[j][0] - h.x, w[j][1] - h.y);
    }
    if constexpr (G <= 4) {
      const uint32_t partner_lo = __shfl_xor_sync(kFull, lo, 16);
      b_hi[j] = g < 4 ? hi : partner_lo;
      b_lo[j] = 0u;
    } else {
      b_hi[j] = hi;
      b_lo[j] = lo;
    }
  }
}

// Write a warp's chain state into the group merge area: m, l per head, acc as [h][dim].
template <int D, int G>
__device__ __forceinline__ void chain_to_smem(float (&acc)[D / 16][4], float m_run, float l_run, float* area_w,
                                             float* m_w, float* l_w, const int (&dim_of)[D / 16][2]) {
  const int lane = threadIdx.x & 31, g = lane >> 2, tq = lane & 3;
  l_run += __shfl_xor_sync(kFull, l_run, 1);
  l_run += __shfl_xor_sync(kFull, l_run, 2);
  if (tq == 0 && g < G) {
    m_w[g] = m_run;
    l_w[g] = l_run;
  }
  if constexpr (G <= 4) {  // fold the residual columns 4..7 into heads 0..3
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[mt][e] += __shfl_xor_sync(kFull, acc[mt][e], 2);
  }
#pragma unroll
  for (int mt = 0; mt < D / 16; ++mt)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int h = 2 * tq + (e & 1);
      if (h < G) area_w[h * D + dim_of[mt][e >> 1]] = acc[mt][e];
    }
}

// Unnormalised Walsh-Hadamard transform, Sylvester order, of a (C * L)-vector held by a
// group of L consecutive lanes, C elements per lane: lane `part` of the group holds elements
// [C part, C part + C).  The stages run in increasing stride: those below C inside the lane,
// the others against lane part ^ (stride / C) of the same group.  Every butterfly is
// (lower + upper, lower - upper), so the result does not depend on C.
template <int C, int L>
__device__ __forceinline__ void group_fwht(float (&x)[C], int part) {
#pragma unroll
  for (int h = 1; h < C; h <<= 1)
#pragma unroll
    for (int j = 0; j < C; ++j)
      if ((j & h) == 0) {
        const float a = x[j], b = x[j + h];
        x[j] = a + b;
        x[j + h] = a - b;
      }
#pragma unroll
  for (int m = 1; m < L; m <<= 1) {
    const bool upper = (part & m) != 0;
#pragma unroll
    for (int j = 0; j < C; ++j) {
      const float o = __shfl_xor_sync(kFull, x[j], m);
      x[j] = upper ? o - x[j] : x[j] + o;
    }
  }
}

__device__ __forceinline__ void sts64(uint32_t a, uint32_t x, uint32_t y) {
  asm volatile("st.shared.v2.b32 [%0], {%1, %2};\n" ::"r"(a), "r"(x), "r"(y) : "memory");
}
__device__ __forceinline__ void sts128(uint32_t a, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};\n" ::"r"(a), "r"(x), "r"(y), "r"(z), "r"(w) : "memory");
}

// Merge the NW chain states of a finished item (group threads) and write its partials.
// First the G per-head statistics and the NW x G chain factors exp2(m_w - M) / L are
// computed once; then every output is one dot product over chains.
template <int D, int G, int NW>
__device__ __forceinline__ void merge_item(const AttendParams& p, const Item& it, int gi, float* area, float* mws,
                                           float* lws, float* fac) {
  const int tg = threadIdx.x - gi * NW * 32;  // thread index within the group
  if (tg < G) {
    const int h = tg;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, mws[w * G + h]);
    float L = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) L = fmaf(lws[w * G + h], exp2f(mws[w * G + h] - M), L);
    const float inv = 1.f / L;
#pragma unroll
    for (int w = 0; w < NW; ++w) fac[w * G + h] = exp2f(mws[w * G + h] - M) * inv;  // 0 for an empty chain
    p.lse_part[(size_t)it.slot * p.Hq + it.kvh * G + h] = kLn2 * (M + log2f(L));
  }
  group_sync<NW>(gi);
  for (int i = tg; i < G * D; i += NW * 32) {
    const int h = i / D, dim = i % D;
    float o = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) o = fmaf(area[(w * G + h) * D + dim], fac[w * G + h], o);
    p.o_part[((size_t)it.slot * p.Hq + it.kvh * G + h) * D + dim] = o;
  }
}

// ------------------------------------------------------------------------------------
// exact BF16 tier
// ------------------------------------------------------------------------------------
template <int D, int G, int NW, int NST>
struct Bf16Cfg {
  static constexpr int HALVES = D / 64;            // 64-element TMA boxes per row
  static constexpr int BOX = 16 * 128;             // one 16-row x 64-element box
  static constexpr int TILE = HALVES * BOX;        // one 16-token K or V tile
  static constexpr int STAGE = 2 * TILE;
  static constexpr int RINGS = NW * NST * STAGE;   // 1024-byte aligned stages
  static constexpr int AREA = NW * G * D;          // floats
  static constexpr int FLOATS = AREA + 3 * NW * G;  // area, m, l, factors
  static constexpr int BAR_OFF = RINGS + FLOATS * 4;
  static constexpr size_t SMEM = BAR_OFF + NW * NST * 8 + 1024;  // + alignment slack
};

// Byte offset, inside a TMA-swizzled tile, of 16-byte chunk c (of D/8) of row r.
__device__ __forceinline__ uint32_t tile_off(int r, int c) {
  return (uint32_t)((c >> 3) * (16 * 128) + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

template <int D, int G, int NW, int NST>
__global__ void __launch_bounds__(NW * 32, 1) attend_bf16_mma(const __grid_constant__ AttendParams p) {
  using C = Bf16Cfg<D, G, NW, NST>;
  constexpr int NG = 1;
  extern __shared__ uint8_t smem_raw[];
  // TMA with 128-byte swizzle wants 1024-byte aligned destinations
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, tq = lane & 3;
  const int gi = 0, w = warp;
  float* area = reinterpret_cast<float*>(smem + C::RINGS);
  float* mws = area + C::AREA;
  float* lws = mws + NW * G;
  float* fac = lws + NW * G;
  const uint32_t ring_s = smem_u32(smem + warp * NST * C::STAGE);
  const uint32_t bar_s = smem_u32(smem + C::BAR_OFF) + warp * NST * 8;

  allow_next_grid();
  int lo, hi;
  cta_range(p.seq.item_base[p.seq.n_seq], lo, hi);
  if (lo >= hi) return;  // the same answer in every thread of the CTA
  __shared__ SeqSmem ss_tab;
  fill_seq_smem(p, &ss_tab);
  __syncthreads();
  const SeqSmem* ss = &ss_tab;

  if (lane == 0) {
    for (int j = 0; j < NST; ++j) mbar_init(bar_s + 8 * j, 1);
    fence_mbar_init();
  }
  __syncwarp();
  wait_prior_grids();  // every global access comes after this

  // paged tiers: lane j holds the page ids of steps j and 32 + j of item pid_slot (one
  // coalesced load per lane when the loader reaches an item)
  int pid0 = 0, pid1 = 0, pid_slot = -1;
  const uint64_t pol = l2_evict_first();
  // lane 0 fills stage st with step s of item it: one TMA box per 64-element half of K and V
  auto load_step = [&](const Item& it, int s, int st) {
    int page = 0;
    if (p.tier.paged) {  // warp-uniform
      if (it.slot != pid_slot) {
        pid_slot = it.slot;
        const int nst = (it.n + 15) >> 4, lp0 = it.t0 >> 4;
        pid0 = lane < nst ? (int)tier_page(p.tier, it.b, lp0 + lane, p.err) : 0;
        pid1 = 32 + lane < nst ? (int)tier_page(p.tier, it.b, lp0 + 32 + lane, p.err) : 0;
      }
      page = __shfl_sync(kFull, s < 32 ? pid0 : pid1, s & 31);
    }
    if (lane == 0) {
      int c1, c3;
      if (p.tier.paged) {
        c1 = 0;
        c3 = page;
      } else {
        c1 = it.t0 + 16 * s;
        c3 = it.b;
      }
      const uint32_t bar = bar_s + 8 * st, dst = ring_s + st * C::STAGE;
      // TMA dimension j + 1 takes logical coordinate tperm[j] (selects, not an indexed
      // array, which would live in local memory)
      auto pick = [&](int j) { return p.tperm[j] == 0 ? c1 : (p.tperm[j] == 1 ? it.kvh : c3); };
      const int x1 = pick(0), x2 = pick(1), x3 = pick(2);
      fence_proxy_async();
      mbar_expect_tx(bar, C::STAGE);
#pragma unroll
      for (int hv = 0; hv < C::HALVES; ++hv) {
        tma_load_4d(dst + hv * C::BOX, &p.tmk, 64 * hv, x1, x2, x3, bar, pol);
        tma_load_4d(dst + C::TILE + hv * C::BOX, &p.tmv, 64 * hv, x1, x2, x3, bar, pol);
      }
    }
  };

  Cursor ld;
  ld.item = lo + gi;
  ld.step = w;
  ld.info = item_at(p, ld.item, ss);
  cursor_settle<NG>(p, ld, hi, w, ss);
  int issued = 0;
#pragma unroll
  for (int j = 0; j < NST; ++j) {
    if (ld.item < hi) {
      load_step(ld.info, ld.step, j);
      cursor_next<NW, NG>(p, ld, hi, w, ss);
      ++issued;
    }
  }

  int dim_of[D / 16][2];
#pragma unroll
  for (int mt = 0; mt < D / 16; ++mt) {
    dim_of[mt][0] = 16 * mt + g;
    dim_of[mt][1] = 16 * mt + 8 + g;
  }
  uint32_t qa[D / 16][4];
  int q_pair = -1;
  int stage = 0;
  uint32_t phases = 0;  // bit j: parity of stage j's next completion
  bool ok = true;

  for (int item = lo + gi; item < hi; item += NG) {
    const Item it = item_at(p, item, ss);
    if (it.pair != q_pair) {  // A fragments of q: rows = heads; rows >= G and 8..15 zero
      q_pair = it.pair;
      const uint16_t* qrow = p.q + ((size_t)it.b * p.Hq + (size_t)it.kvh * G + (g < G ? g : 0)) * D;
#pragma unroll
      for (int kc = 0; kc < D / 16; ++kc) {
        const uint32_t a = *reinterpret_cast<const uint32_t*>(qrow + 16 * kc + 2 * tq);
        const uint32_t b = *reinterpret_cast<const uint32_t*>(qrow + 16 * kc + 8 + 2 * tq);
        qa[kc][0] = g < G ? a : 0u;
        qa[kc][1] = 0u;
        qa[kc][2] = g < G ? b : 0u;
        qa[kc][3] = 0u;
      }
    }
    float acc[D / 16][4];
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[mt][e] = 0.f;
    float m_run = -INFINITY, l_run = 0.f;

    for (int s = w; 16 * s < it.n; s += NW) {
      if (ok) ok = __all_sync(kFull, mbar_wait(bar_s + 8 * stage, (phases >> stage) & 1u));  // warp-uniform
      phases ^= 1u << stage;
      --issued;
      if (ok) {
        const int nv = min(16, it.n - 16 * s);
        const uint32_t kt = ring_s + stage * C::STAGE, vt = kt + C::TILE;
        uint8_t* vt_g = smem + warp * NST * C::STAGE + stage * C::STAGE + C::TILE;
        if (nv < 16) {  // rows past the split may hold anything: clear them in V
          for (int i = lane; i < (16 - nv) * C::HALVES * 8; i += 32) {
            const int r = nv + i / (C::HALVES * 8), rem = i % (C::HALVES * 8);
            *reinterpret_cast<uint4*>(vt_g + (rem >> 3) * C::BOX + r * 128 + (rem & 7) * 16) = make_uint4(0, 0, 0, 0);
          }
          __syncwarp();
        }
        float sc[2][4];
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
          for (int e = 0; e < 4; ++e) sc[j][e] = 0.f;
#pragma unroll
        for (int kc = 0; kc < D / 16; ++kc) {
          const int mi = lane >> 3, r = (mi >> 1) * 8 + (lane & 7), c = 2 * kc + (mi & 1);
          uint32_t b[4];
          ldsm_x4(b, kt + tile_off(r, c));
          mma_bf16(sc[0], qa[kc], b[0], b[1]);
          mma_bf16(sc[1], qa[kc], b[2], b[3]);
        }
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
          for (int e = 0; e < 2; ++e) sc[j][e] *= p.scale_log2;
        if (nv < 16) {
#pragma unroll
          for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int e = 0; e < 2; ++e)
              if (8 * j + 2 * tq + e >= nv) sc[j][e] = -INFINITY;
        }
        float a_even, a_odd;
        if (online_softmax<G>(sc, m_run, l_run, a_even, a_odd)) {
#pragma unroll
          for (int mt = 0; mt < D / 16; ++mt) {
            acc[mt][0] *= a_even; acc[mt][1] *= a_odd;
            acc[mt][2] *= a_even; acc[mt][3] *= a_odd;
          }
        }
        const float wts[2][2] = {{sc[0][0], sc[0][1]}, {sc[1][0], sc[1][1]}};
        uint32_t pb[2], pl[2];
        p_fragments<G, true>(wts, pb, pl);
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) {
          const int mi = lane >> 3, r = (mi >> 1) * 8 + (lane & 7), c = 2 * mt + (mi & 1);
          uint32_t a[4];
          ldsm_x4_t(a, vt + tile_off(r, c));
          mma_bf16(acc[mt], a, pb[0], pb[1]);
          if constexpr (G > 4) mma_bf16(acc[mt], a, pl[0], pl[1]);
        }
        __syncwarp();
        if (ld.item < hi) {
          load_step(ld.info, ld.step, stage);
          cursor_next<NW, NG>(p, ld, hi, w, ss);
          ++issued;
        }
      }
      stage = stage + 1 == NST ? 0 : stage + 1;
    }
    chain_to_smem<D, G>(acc, m_run, l_run, area + w * G * D, mws + w * G, lws + w * G, dim_of);
    group_sync<NW>(gi);
    merge_item<D, G, NW>(p, it, gi, area, mws, lws, fac);
    group_sync<NW>(gi);
  }
  if (!ok) {
    // a wait ran out: record it, then give the copies still in flight a bounded chance
    // to land before the CTA's shared memory goes away
    if (lane == 0) flag_error(p.err, AKV_EFLAG_TIMEOUT);
    for (; issued > 0; --issued) {
      mbar_wait(bar_s + 8 * stage, (phases >> stage) & 1u);
      phases ^= 1u << stage;
      stage = stage + 1 == NST ? 0 : stage + 1;
    }
  }
}

// ------------------------------------------------------------------------------------
// compact tier (CODES4): one warp per split
// ------------------------------------------------------------------------------------
// Every split of the compact tier is one chain: a single warp runs all of its 16-token
// steps in order, so the split needs no cross-warp merge.  The grid is persistent (one CTA
// of NWARP warps per SM) and every warp owns an equal contiguous range of items.
//
// Shared memory.  The lookup table is 256 rows of 256 bytes at the first 64 KB boundary of
// the CTA's window: entry b for lane l sits at table + 256 b + 4 l and holds the half pair
// (c[b & 15], c[b >> 4]).  One copy per lane keeps the gathers conflict-free, and with the
// table 64 KB aligned one byte permute of (code word, table | 4 lane) yields the entry's
// full shared address.  The upper 128 bytes of every table row are each warp's scratch
// (G x D words for the query and output rotations, SCR_ROWS rows per warp).  Each warp's
// ring of NST stages sits below the table while they fit and above it after.  A stage
// holds one 16-token key block and one value block exactly as stored, filled by cp.async.
// The value block's pair-row layout (byte k of pair row r = code k of tokens 2r, 2r + 1;
// unit u of D/8 bytes at position u ^ w(r)) is the A-fragment order of the value product,
// and its unit swizzle makes the fragment reads conflict-free.
template <int D, int G, int NWARP, int NST>
struct CodesCfg {
  static constexpr int ROWB = D / 2;
  static constexpr int BLOCK = AKV_CODES4_BLOCK_BYTES(D);
  static constexpr int K_OFF = 0;                  // the key block as stored
  static constexpr int KS_OFF = 16 * ROWB;
  static constexpr int V_OFF = BLOCK;              // the value block as stored
  static constexpr int VS_OFF = BLOCK + 16 * ROWB;
  static constexpr int US = D / 8;                 // value unit: one lane group's dims
  static constexpr int STAGE = 2 * BLOCK;
  static constexpr int LUT = 1 << 16;
  static constexpr int SCR_ROWS = G * D / 32;
  static constexpr int PER_WARP = NST * STAGE;
  // Wherever the window starts, the rings below the table waste less than one ring, and
  // an all-below layout ends within two table lengths of the start.
  static constexpr int SPAN = NWARP * PER_WARP + PER_WARP;
  static constexpr size_t SMEM = (size_t)LUT + (size_t)(SPAN > LUT ? SPAN : LUT);
  static_assert(SCR_ROWS * NWARP <= 256, "scratch fits the table rows' upper halves");
  static_assert(PER_WARP % 16 == 0 && STAGE % 16 == 0, "16-byte aligned rings and stages");
  static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
};

// Where the table and this warp's ring sit; false when the launch's dynamic shared memory
// is too small for the layout (the caller flags it and does nothing).
template <class C, int NWARP>
__device__ __forceinline__ bool codes_layout(uint32_t base_s, int warp, uint32_t& lut_s, uint32_t& ring_s) {
  lut_s = (base_s + 0xFFFFu) & ~0xFFFFu;
  const int below = min(NWARP, (int)((lut_s - base_s) / C::PER_WARP));
  const uint32_t top = lut_s + C::LUT + (uint32_t)(NWARP - below) * C::PER_WARP;
  uint32_t dyn;
  asm("mov.u32 %0, %%dynamic_smem_size;\n" : "=r"(dyn));
  ring_s = warp < below ? base_s + warp * C::PER_WARP : lut_s + C::LUT + (warp - below) * C::PER_WARP;
  return top - base_s <= dyn;
}

__device__ __forceinline__ void sts32(uint32_t a, uint32_t v) {
  asm volatile("st.shared.b32 [%0], %1;\n" ::"r"(a), "r"(v) : "memory");
}

template <int D, int G, int NWARP, int NST>
__global__ void __launch_bounds__(NWARP * 32, 1) attend_codes_mma(const __grid_constant__ AttendParams p) {
  using C = CodesCfg<D, G, NWARP, NST>;
  constexpr int DPT = D / 8;                      // value dims per lane group
  constexpr int KB = D / 8;                       // key code bytes per lane
  // rotations (query in, output out): lane group qh of LPH lanes holds head qh, CPL
  // coordinates per lane, so the transform needs log2(LPH) shuffle stages, not 5
  constexpr int LPH = 32 / G, CPL = D / LPH;
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, tq = lane & 3;
  const int qh = lane / LPH, qp = lane % LPH;  // this lane's head and part in the rotations
  const uint32_t base_s = smem_u32(smem);
  uint32_t lut_s, ring_s;
  allow_next_grid();
  if (!codes_layout<C, NWARP>(base_s, warp, lut_s, ring_s)) {  // same answer in every thread
    wait_prior_grids();
    if (threadIdx.x == 0) flag_error(p.err, AKV_EFLAG_INTERNAL);
    return;
  }
  // word i of this warp's scratch: in the upper half of its table row r = i / 32, at word
  // (i % 32) ^ 4 (r % 8) -- the 16-byte units of a row are XOR-swizzled by the row, so the
  // query-fragment reads and the rotation reads are conflict-free and the output writes
  // at most 2-way
  const uint32_t scr_s = lut_s + (uint32_t)(warp * C::SCR_ROWS) * 256u + 128u;
  auto scr = [&](int i) -> uint32_t {
    const uint32_t r = (uint32_t)i >> 5;
    return scr_s + (r << 8) + ((((uint32_t)i & 31u) ^ ((r & 7u) << 2)) << 2);
  };

  // this warp's item range: an equal share of all items, in item order; warps are numbered
  // warp-major across CTAs so a partly filled grid still spreads its busy warps over every SM
  const int total = p.seq.item_base[p.seq.n_seq];
  const int nw = (int)gridDim.x * NWARP, gw = warp * (int)gridDim.x + (int)blockIdx.x;
  const int q0 = total / nw, r0 = total % nw;
  const int lo = gw * q0 + min(gw, r0), hi = lo + q0 + (gw < r0 ? 1 : 0);
  const bool busy = lo < hi;

  // the query coordinates [CPL qp, CPL qp + CPL) of head qh, as bf16 pairs; the first item's
  // are requested before anything else so their latency hides behind the stage loads and
  // the table build
  auto load_q = [&](const Item& it, uint32_t (&qw)[CPL / 2]) {
    const uint16_t* qrow = p.q + ((size_t)it.b * p.Hq + (size_t)it.kvh * G + qh) * D + CPL * qp;
    if constexpr (CPL >= 8) {
#pragma unroll
      for (int i = 0; i < CPL / 8; ++i) {
        const uint4 v = reinterpret_cast<const uint4*>(qrow)[i];
        qw[4 * i] = v.x; qw[4 * i + 1] = v.y; qw[4 * i + 2] = v.z; qw[4 * i + 3] = v.w;
      }
    } else if constexpr (CPL == 4) {
      const uint2 v = *reinterpret_cast<const uint2*>(qrow);
      qw[0] = v.x;
      qw[1] = v.y;
    } else {
      qw[0] = *reinterpret_cast<const uint32_t*>(qrow);
    }
  };
  // the lookup table is built from the launch parameters, before the wait for the previous
  // grid; every global access comes after it
  {
    uint32_t* lut = reinterpret_cast<uint32_t*>(smem + (lut_s - base_s));
    for (int i = threadIdx.x; i < 256 * 32; i += NWARP * 32) {
      const int byte = i >> 5, l = i & 31;
      lut[byte * 64 + l] = (uint32_t)p.centroids[byte & 15] | ((uint32_t)p.centroids[byte >> 4] << 16);
    }
  }
  // the sequence table goes to shared memory with the lookup table; both are complete after
  // the block-wide barrier below, so the loader's first item reads the parameters
  __shared__ SeqSmem ss_tab;
  fill_seq_smem(p, &ss_tab);
  const SeqSmem* ss = nullptr;
  wait_prior_grids();
  uint32_t qw[CPL / 2];
  if (busy) load_q(item_at(p, lo, nullptr), qw);

  // ---- loader: the (item, step) of the next stage to fill.  Global step S of this warp
  // (counted over its items) uses stage S % NST.  The lanes copy the key block and the value
  // block into it as stored, in 16-byte chunks (lane l: chunks l, l + 32, l + 64 of each
  // that exist), as one cp.async commit group per step.
  constexpr int CH = C::BLOCK / 16;  // 16-byte chunks per block
  static_assert(CH > 32 && CH <= 96, "at most three chunk rounds per block");
  int ld_item = lo, ld_left = 0;  // the loader's item and its steps not yet issued
  int ld_step = 0;                 // the step of that item the loader issues next
  // paged tiers: lane j holds the page ids of the item's steps j and 32 + j, loaded (one
  // coalesced load per lane) when the loader reaches the item, so issuing a step needs a
  // shuffle instead of a dependent global load
  int ld_pid0 = 0, ld_pid1 = 0;
  // contiguous tiers: this lane's first chunk of the next key block, stepped by one token
  // block per step; paged tiers: of the head's block in page 0.  A value block sits at a
  // fixed distance from its key block.
  const uint8_t* ld_k = nullptr;
  const int64_t kv_delta = (int64_t)((uintptr_t)p.tier.v - (uintptr_t)p.tier.k);
  const int64_t step_bytes = p.tier.s_tok * (int64_t)C::BLOCK;
  const uint32_t lane16 = 16u * (uint32_t)lane;
  auto ld_begin = [&]() {
    const Item it = item_at(p, ld_item, ss);
    ld_left = (it.n + 15) >> 4;
    ld_step = 0;
    const int lp0 = it.t0 >> 4;
    int64_t blk = (int64_t)it.kvh * p.tier.s_head;
    if (p.tier.paged) {
      ld_pid0 = lane < ld_left ? (int)tier_page(p.tier, it.b, lp0 + lane, p.err) : 0;
      ld_pid1 = 32 + lane < ld_left ? (int)tier_page(p.tier, it.b, lp0 + 32 + lane, p.err) : 0;
    } else {
      blk += (int64_t)it.b * p.tier.s_seq + (int64_t)lp0 * p.tier.s_tok;
    }
    ld_k = p.tier.k + blk * C::BLOCK + lane16;
  };
  auto ld_issue = [&](uint32_t stage_s) {  // fills the stage at shared address stage_s
    const uint64_t pol = l2_evict_first();
    const uint8_t* kb = ld_k;
    if (p.tier.paged) {
      const int64_t page = __shfl_sync(kFull, ld_step < 32 ? ld_pid0 : ld_pid1, ld_step & 31);
      kb += page * p.tier.s_seq * (int64_t)C::BLOCK;
    } else {
      ld_k += step_bytes;
    }
    const uint8_t* vb = kb + kv_delta;
    const uint32_t dst = stage_s + lane16;
    cp_async16(dst + C::K_OFF, kb, pol);
    cp_async16(dst + C::V_OFF, vb, pol);
    if (CH >= 64 || 32 + lane < CH) {
      cp_async16(dst + C::K_OFF + 512, kb + 512, pol);
      cp_async16(dst + C::V_OFF + 512, vb + 512, pol);
    }
    if (64 + lane < CH) {
      cp_async16(dst + C::K_OFF + 1024, kb + 1024, pol);
      cp_async16(dst + C::V_OFF + 1024, vb + 1024, pol);
    }
    ++ld_step;
    if (--ld_left == 0 && ++ld_item < hi) ld_begin();
  };
  if (busy) {
    ld_begin();
#pragma unroll
    for (int j = 0; j < NST; ++j) {
      if (ld_item < hi) ld_issue(ring_s + j * C::STAGE);
      cp_async_commit();
    }
  }

  __syncthreads();  // the lookup table and the sequence table are complete
  if (!busy) return;
  ss = &ss_tab;

  // table entry of byte `byte` of `word` for this lane: the table's own high address bytes,
  // the code byte as bits 8..15 and 4 lane as bits 0..7, assembled by one byte permute
  const uint32_t lane4 = lut_s | ((uint32_t)lane << 2);
  auto lookup = [&](uint32_t word, int byte) -> uint32_t {
    return lds32_const(__byte_perm(word, lane4, 0x7604 | (byte << 4)));
  };
  // this lane's offsets inside a stage: key code bytes [KB tq, KB tq + KB) of token g (+ 8),
  // the scales of tokens 2tq, 2tq + 1 (+ 8), value code bytes of dims [DPT g, DPT g + DPT)
  // of tokens 2tq, 2tq + 1 (+ 8)
  const uint32_t koff = C::K_OFF + g * C::ROWB + KB * tq;
  const uint32_t ksoff = C::KS_OFF + 2 * g;  // token g's key scale; the value scales sit at + VS_OFF - KS_OFF
  const uint32_t voff = C::V_OFF + tq * D + C::US * (g ^ (D == 128 ? 2 * tq : 4 * (tq >> 1)));
  static_assert((NST & (NST - 1)) == 0, "stage index by mask");
  int gs = 0;  // this warp's global step; its stage is gs % NST

  // Score columns: G <= 4 -- column c < 4 is head c's high part, column c + 4 its residual;
  // G = 8 -- columns are the heads, the residuals in a second product.  Lane (g, tq) holds
  // the scores of heads hA = 2tq, hB = 2tq + 1 (mod 4 when G <= 4) at tokens g and g + 8;
  // when G <= 4 lanes tq >= 2 duplicate lanes tq - 2.
  constexpr int NQ = G <= 4 ? 1 : 2;
  const int hA = G <= 4 ? (2 * tq) & 3 : 2 * tq, hB = hA + 1;
  uint32_t qb[NQ][D / 16][2];  // B fragments of the query columns
  float kfA = 0.f, kfB = 0.f;  // score factors of heads hA, hB
  int q_pair = -1;

  // Base-2 scores of the step held in stage sa: sc[t][e] is head (hA, hB)[e] at token g + 8t.
  // S (16 tokens x 8 columns) = K_hat Q^T: the A fragments (tokens g and g + 8 over the
  // lane's dimension range) are looked up straight from the key code bytes and accumulated
  // as two independent chains (even and odd 16-dimension slices, so the products overlap);
  // the chains, then the high and residual columns are added, then the key scale applied.
  auto scores = [&](uint32_t sa, float (&sc)[2][2]) {
    uint32_t wk[2][KB / 4];
    const uint32_t ka = sa + koff;
    if constexpr (KB == 16) {
      const uint4 a = lds128<0>(ka), b = lds128<8 * C::ROWB>(ka);
      wk[0][0] = a.x; wk[0][1] = a.y; wk[0][2] = a.z; wk[0][3] = a.w;
      wk[1][0] = b.x; wk[1][1] = b.y; wk[1][2] = b.z; wk[1][3] = b.w;
    } else {
      const uint2 a = lds64<0>(ka), b = lds64<8 * C::ROWB>(ka);
      wk[0][0] = a.x; wk[0][1] = a.y;
      wk[1][0] = b.x; wk[1][1] = b.y;
    }
    float st[NQ][4], st_odd[NQ][4];
#pragma unroll
    for (int q = 0; q < NQ; ++q)
#pragma unroll
      for (int e = 0; e < 4; ++e) st[q][e] = st_odd[q][e] = 0.f;
#pragma unroll
    for (int kc = 0; kc < D / 16; ++kc) {
      const uint32_t w0 = wk[0][kc >> 1], w1 = wk[1][kc >> 1];
      const int bt = 2 * (kc & 1);
      const uint32_t a[4] = {lookup(w0, bt), lookup(w1, bt), lookup(w0, bt + 1), lookup(w1, bt + 1)};
#pragma unroll
      for (int q = 0; q < NQ; ++q) mma_f16((kc & 1) ? st_odd[q] : st[q], a, qb[q][kc][0], qb[q][kc][1]);
    }
#pragma unroll
    for (int q = 0; q < NQ; ++q)
#pragma unroll
      for (int e = 0; e < 4; ++e) st[q][e] += st_odd[q][e];
    float v[4];
#pragma unroll
    for (int e = 0; e < 4; ++e)
      v[e] = NQ == 1 ? st[0][e] + __shfl_xor_sync(kFull, st[0][e], 2) : st[0][e] + st[NQ - 1][e];
    const float ks0 = lds_half<0>(sa + ksoff), ks8 = lds_half<16>(sa + ksoff);
    sc[0][0] = v[0] * (kfA * ks0);
    sc[0][1] = v[1] * (kfB * ks0);
    sc[1][0] = v[2] * (kfA * ks8);
    sc[1][1] = v[3] * (kfB * ks8);
  };

  for (int item = lo; item < hi; ++item) {
    const Item it = item_at(p, item, ss);
    if (it.pair != q_pair) {
      if (item != lo) load_q(it, qw);
      q_pair = it.pair;
      // rotate: lane group qh transforms head qh (the tier's rotation signs first), scales it
      // by a power of two to [0.5, 1) and writes the FP16 (high, residual) words of its dims
      // (2i, 2i + 1) to scratch words qh D + 2i and qh D + 2i + 1
      float x[CPL];
#pragma unroll
      for (int j = 0; j < CPL / 2; ++j) {
        x[2 * j] = bf16lo(qw[j]) * coord_sign(p.tier, CPL * qp + 2 * j);
        x[2 * j + 1] = bf16hi(qw[j]) * coord_sign(p.tier, CPL * qp + 2 * j + 1);
      }
      group_fwht<CPL, LPH>(x, qp);
      float mx = 0.f;
#pragma unroll
      for (int j = 0; j < CPL; ++j) mx = fmaxf(mx, fabsf(x[j]));
#pragma unroll
      for (int m = 1; m < LPH; m <<= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, m));
      __syncwarp();  // earlier reads of the scratch are done
      int e = 0;
      if (mx > 0.f) frexpf(mx, &e);
      const float inv = ldexpf(1.f, -e);
      uint32_t wq[CPL];
#pragma unroll
      for (int j = 0; j < CPL; j += 2) {
        const float x0 = x[j] * inv, x1 = x[j + 1] * inv;
        wq[j] = pack_f16(x0, x1);
        const float2 hv = unpack_f16(wq[j]);
        wq[j + 1] = pack_f16(x0 - hv.x, x1 - hv.y);
      }
      if constexpr (CPL >= 4) {
#pragma unroll
        for (int j = 0; j < CPL; j += 4) sts128(scr(qh * D + CPL * qp + j), wq[j], wq[j + 1], wq[j + 2], wq[j + 3]);
      } else {
        sts64(scr(qh * D + CPL * qp), wq[0], wq[1]);
      }
      // the scale exponents of this lane's score heads hA, hB (heads >= G give 0; their
      // columns are never stored)
      const int eA_src = hA < G ? hA : 0, eB_src = hB < G ? hB : 0;
      const int eA_g = __shfl_sync(kFull, e, eA_src * LPH), eB_g = __shfl_sync(kFull, e, eB_src * LPH);
      const int eA = hA < G ? eA_g : 0, eB = hB < G ? eB_g : 0;
      __syncwarp();
      // column g, step kc: dims 2*KB*tq + 4kc + {0, 1} (b0) and + {2, 3} (b1) of the lane's
      // k range; the scratch holds (high, residual) word pairs per two dims
      const int hg = G <= 4 ? (g & 3) : g;
      const bool on = hg < G;
      const int i0 = (on ? hg : 0) * D + 2 * KB * tq;
#pragma unroll
      for (int kc = 0; kc < D / 16; ++kc) {
        const uint4 v = lds128<0>(scr(i0 + 4 * kc));
        if constexpr (NQ == 1) {
          const bool lo_part = g >= 4;
          qb[0][kc][0] = on ? (lo_part ? v.y : v.x) : 0u;
          qb[0][kc][1] = on ? (lo_part ? v.w : v.z) : 0u;
        } else {
          qb[0][kc][0] = v.x;
          qb[0][kc][1] = v.z;
          qb[NQ - 1][kc][0] = v.y;
          qb[NQ - 1][kc][1] = v.w;
        }
      }
      kfA = p.scale_log2 / (float)D * ldexpf(1.f, eA);
      kfB = p.scale_log2 / (float)D * ldexpf(1.f, eB);
      __syncwarp();
    }

    float acc[D / 16][4];
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[mt][e] = 0.f;
    float m_A = -INFINITY, m_B = -INFINITY, l_A = 0.f, l_B = 0.f;  // heads hA, hB
    const int nsteps = (it.n + 15) >> 4;
    // Commit groups are counted in steps: before step S of this warp NST + S groups have been
    // committed, so waiting down to NST - 1 pending lands step S, and down to NST - 2 lands
    // step S + 1 as well.
    float sc_n[2][2];
    cp_async_wait<NST - 1>();
    __syncwarp();
    scores(ring_s + (gs & (NST - 1)) * C::STAGE, sc_n);

#pragma unroll 2  // fewer per-step moves and stage bookkeeping (measured)
    for (int s = 0; s < nsteps; ++s) {
      cp_async_wait<NST - 2>();  // this step and the next have landed
      __syncwarp();
      const uint32_t st_s = ring_s + (gs & (NST - 1)) * C::STAGE;
      const uint32_t nxt = ring_s + ((gs + 1) & (NST - 1)) * C::STAGE;
      float sc[2][2] = {{sc_n[0][0], sc_n[0][1]}, {sc_n[1][0], sc_n[1][1]}};
      const int nv = min(16, it.n - 16 * s);
      if (nv < 16) {
#pragma unroll
        for (int t = 0; t < 2; ++t)
          if (g + 8 * t >= nv) sc[t][0] = sc[t][1] = -INFINITY;
      }
      // the next step's scores, so their loads, lookups and MMAs overlap this step's
      // softmax and value product (after an item's last step the next stage holds the
      // following item's first step or nothing; those scores are not used)
      scores(nxt, sc_n);
      // ---- online softmax per head over the 16 tokens (2 per lane, 8 lane groups).  The
      // reference m of each head sits kSlack above a maximum already seen, so the weights
      // 2^(s - m) stay at most 1; only a score above m (in practice a split's first steps)
      // costs the cross-lane maximum and the rescale.  LSE = m + log2 l holds for any m.
      constexpr float kSlack = 8.f;
      float mxA = fmaxf(sc[0][0], sc[1][0]), mxB = fmaxf(sc[0][1], sc[1][1]);
      if (__any_sync(kFull, mxA > m_A || mxB > m_B)) {
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
          mxA = fmaxf(mxA, __shfl_xor_sync(kFull, mxA, off));
          mxB = fmaxf(mxB, __shfl_xor_sync(kFull, mxB, off));
        }
        const float nA = fmaxf(m_A, mxA + kSlack), nB = fmaxf(m_B, mxB + kSlack);
        const float aA = fast_exp2(m_A - nA), aB = fast_exp2(m_B - nB);  // 0 while m = -inf
        l_A *= aA;
        l_B *= aB;
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) {  // accumulator columns 2tq, 2tq + 1 are heads hA, hB
          acc[mt][0] *= aA; acc[mt][1] *= aB;
          acc[mt][2] *= aA; acc[mt][3] *= aB;
        }
        m_A = nA;
        m_B = nB;
      }
      float w[2][2];
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        w[t][0] = fast_exp2(sc[t][0] - m_A);
        w[t][1] = fast_exp2(sc[t][1] - m_B);
      }
      l_A += w[0][0] + w[1][0];
      l_B += w[0][1] + w[1][1];
      // ---- P' = P * s^V as the value product's B fragments.  Lane (g, tq) holds P' of tokens
      // g, g + 8 at columns 2tq, 2tq + 1 (G <= 4: lanes tq < 2 the FP16 high parts, tq >= 2 the
      // residuals); a transpose per 8 tokens gives column g at tokens 2tq, 2tq + 1 (+ 8).
      const float vs0 = lds_half<C::VS_OFF - C::KS_OFF>(st_s + ksoff);
      const float vs8 = lds_half<C::VS_OFF - C::KS_OFF + 16>(st_s + ksoff);
      w[0][0] *= vs0; w[0][1] *= vs0;
      w[1][0] *= vs8; w[1][1] *= vs8;
      if (nv < 16) {
#pragma unroll
        for (int t = 0; t < 2; ++t)
          if (g + 8 * t >= nv) w[t][0] = w[t][1] = 0.f;
      }
      uint32_t pb[2], pl[2];
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const uint32_t hi = pack_f16(w[t][0], w[t][1]);
        const float2 hv = unpack_f16(hi);
        const uint32_t lo = pack_f16(w[t][0] - hv.x, w[t][1] - hv.y);
        if constexpr (NQ == 1) {
          pb[t] = transpose8x8(tq >= 2 ? lo : hi);
          pl[t] = 0u;
        } else {
          pb[t] = transpose8x8(hi);
          pl[t] = transpose8x8(lo);
        }
      }
      // ---- O_rot^T += V_hat^T P'^T: lane (g, tq) reads value dims [DPT g, DPT g + DPT) of
      // token pairs (2tq, 2tq+1) (pair row tq) and (2tq+8, 2tq+9) (pair row 4 + tq); byte k
      // of those words is dim DPT g + k of both tokens, so one lookup is one A-fragment entry
      uint32_t vw[2][DPT / 4];
      const uint32_t va = st_s + voff;
      if constexpr (DPT == 16) {
        const uint4 a = lds128<0>(va), b = lds128<4 * D>(va);
        vw[0][0] = a.x; vw[0][1] = a.y; vw[0][2] = a.z; vw[0][3] = a.w;
        vw[1][0] = b.x; vw[1][1] = b.y; vw[1][2] = b.z; vw[1][3] = b.w;
      } else {
        const uint2 a = lds64<0>(va), b = lds64<4 * D>(va);
        vw[0][0] = a.x; vw[0][1] = a.y;
        vw[1][0] = b.x; vw[1][1] = b.y;
      }
#pragma unroll
      for (int mt = 0; mt < D / 16; ++mt) {
        uint32_t a[4];
        const int m0 = mt, m1 = DPT / 2 + mt;  // rows g and g + 8 of this 16-dim tile
        a[0] = lookup(vw[0][m0 >> 2], m0 & 3);
        a[1] = lookup(vw[0][m1 >> 2], m1 & 3);
        a[2] = lookup(vw[1][m0 >> 2], m0 & 3);
        a[3] = lookup(vw[1][m1 >> 2], m1 & 3);
        mma_f16(acc[mt], a, pb[0], pb[1]);
        if constexpr (G > 4) mma_f16(acc[mt], a, pl[0], pl[1]);
      }
      __syncwarp();
      if (ld_item < hi) ld_issue(st_s);  // refills the stage just read
      cp_async_commit();
      ++gs;
    }

    // ---- epilogue: l per head over the 8 lane groups, O = s . H (acc / l) / D per head,
    // LSE = ln 2 (m + log2 l)
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      l_A += __shfl_xor_sync(kFull, l_A, off);
      l_B += __shfl_xor_sync(kFull, l_B, off);
    }
    if (g == 0 && (G > 4 || tq < 2)) {
      float* lse = p.lse_part + (size_t)it.slot * p.Hq + it.kvh * G;
      if (hA < G) lse[hA] = kLn2 * (m_A + log2f(l_A));
      if (hB < G) lse[hB] = kLn2 * (m_B + log2f(l_B));
    }
    const float f_even = 1.f / ((float)D * l_A), f_odd = 1.f / ((float)D * l_B);
    if constexpr (G <= 4) {  // fold the residual columns 4..7 into heads 0..3
#pragma unroll
      for (int mt = 0; mt < D / 16; ++mt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[mt][e] += __shfl_xor_sync(kFull, acc[mt][e], 2);
    }
    __syncwarp();
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int h = 2 * tq + (e & 1);
        const int dim = DPT * g + ((e >> 1) ? DPT / 2 : 0) + mt;
        if (h < G) sts32(scr(h * D + dim), __float_as_uint(acc[mt][e] * ((e & 1) ? f_odd : f_even)));
      }
    __syncwarp();
    {  // lane group qh rotates head qh back and stores it
      float x[CPL];
      if constexpr (CPL >= 4) {
#pragma unroll
        for (int j = 0; j < CPL; j += 4) {
          const uint4 v = lds128<0>(scr(qh * D + CPL * qp + j));
          x[j] = __uint_as_float(v.x); x[j + 1] = __uint_as_float(v.y);
          x[j + 2] = __uint_as_float(v.z); x[j + 3] = __uint_as_float(v.w);
        }
      } else {
        const uint2 v = lds64<0>(scr(qh * D + CPL * qp));
        x[0] = __uint_as_float(v.x); x[1] = __uint_as_float(v.y);
      }
      group_fwht<CPL, LPH>(x, qp);
#pragma unroll
      for (int j = 0; j < CPL; ++j) x[j] *= coord_sign(p.tier, CPL * qp + j);  // undo the rotation signs
      float* dst = p.o_part + ((size_t)it.slot * p.Hq + it.kvh * G + qh) * D + CPL * qp;
      if constexpr (CPL >= 4) {
#pragma unroll
        for (int j = 0; j < CPL; j += 4) *reinterpret_cast<float4*>(dst + j) = make_float4(x[j], x[j + 1], x[j + 2], x[j + 3]);
      } else {
        *reinterpret_cast<float2*>(dst) = make_float2(x[0], x[1]);
      }
    }
    __syncwarp();
  }
  cp_async_wait<0>();
}

template <int D, int G>
cudaError_t launch_bf16(const AttendParams& p, int n_items, cudaStream_t s, int max_ctas, bool overlap) {
  constexpr int NW = 8;
  constexpr int NST = G <= 4 ? 3 : 2;
  using C = Bf16Cfg<D, G, NW, NST>;
  auto k = attend_bf16_mma<D, G, NW, NST>;
  cudaError_t e = ensure_smem<attend_bf16_mma<D, G, NW, NST>>((int)C::SMEM);
  if (e != cudaSuccess) return e;
  const int ctas = max_ctas > 0 ? max_ctas : sm_count();
  const int grid = n_items < ctas ? n_items : ctas;
  e = overlap ? launch_overlapped(k, dim3(grid), dim3(NW * 32), C::SMEM, s, p)
              : (k<<<grid, NW * 32, C::SMEM, s>>>(p), cudaSuccess);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int D, int G>
cudaError_t launch_codes(const AttendParams& p, int n_items, cudaStream_t s, int max_ctas, bool overlap) {
  constexpr int NWARP = G <= 4 ? 16 : 8;
  constexpr int NST = 4;
  using C = CodesCfg<D, G, NWARP, NST>;
  auto k = attend_codes_mma<D, G, NWARP, NST>;
  cudaError_t e = ensure_smem<attend_codes_mma<D, G, NWARP, NST>>((int)C::SMEM);
  if (e != cudaSuccess) return e;
  const int ctas = max_ctas > 0 ? max_ctas : sm_count();
  const int grid = n_items < ctas ? n_items : ctas;
  e = overlap ? launch_overlapped(k, dim3(grid), dim3(NWARP * 32), C::SMEM, s, p)
              : (k<<<grid, NWARP * 32, C::SMEM, s>>>(p), cudaSuccess);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_d(const AttendParams& p, int G, int kind, int n_items, cudaStream_t s, int max_ctas, bool overlap) {
  if (kind == AKV_TIER_BF16) {
    switch (G) {
      case 1: return launch_bf16<D, 1>(p, n_items, s, max_ctas, overlap);
      case 2: return launch_bf16<D, 2>(p, n_items, s, max_ctas, overlap);
      case 4: return launch_bf16<D, 4>(p, n_items, s, max_ctas, overlap);
      default: return launch_bf16<D, 8>(p, n_items, s, max_ctas, overlap);
    }
  }
  switch (G) {
    case 1: return launch_codes<D, 1>(p, n_items, s, max_ctas, overlap);
    case 2: return launch_codes<D, 2>(p, n_items, s, max_ctas, overlap);
    case 4: return launch_codes<D, 4>(p, n_items, s, max_ctas, overlap);
    default: return launch_codes<D, 8>(p, n_items, s, max_ctas, overlap);
  }
}

}  // namespace

// n_items counts (split, KV head) items: seq.item_base must count splits * Hkv.
cudaError_t launch_attend_mma(const AttendParams& p, int d, int G, int kind, int n_items, cudaStream_t s, int max_ctas,
                              bool overlap) {
  return d == 128 ? launch_d<128>(p, G, kind, n_items, s, max_ctas, overlap)
                  : launch_d<64>(p, G, kind, n_items, s, max_ctas, overlap);
}

int codes_warps_per_cta(int G) { return G <= 4 ? 16 : 8; }

}  // namespace akv

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
// Launch.  The grid is persistent: at most one CTA per SM (two groups of NW warps for the
// compact tier), each owning a contiguous, equal-length range of items (item order is
// sequence, then KV head, then split, so consecutive items share their query).  Warp w of
// a group runs chain w of every item of the group back to back through a private ring of
// NST shared-memory stages filled by cp.async; the ring keeps prefetching across item
// boundaries while the group merges the finished item.
//
// Exact BF16 tier, per step (16 tokens):
//   S^T (16 rows x 16 tokens) = q . K^T     A = q rows (heads), B = K rows via ldmatrix
//   O^T (d x 8 cols)         += V^T . P^T   A = V via ldmatrix.trans, B = P from the S^T
//                                           accumulator registers
// The weights P carry a BF16 high part and a BF16 residual: for G <= 4 the residual of
// head h rides in PV column 4 + h of the same MMA, for G = 8 in a second MMA.
// Shared-memory tiles are XOR-swizzled in 16-byte chunks so ldmatrix is conflict-free.
//
// Compact tier, per step: the same contractions in the rotated basis ("QuantForge V2
// Walkthrough", section 1: rotate the query instead of the keys) with FP16 operands.  The
// rotated query H q is split into an FP16 high part (S^T rows 0..7) and residual (rows
// 8..15), so scores keep ~22 significant bits.  Code bytes become (c[lo], c[hi]) half
// pairs through a per-lane replicated table in shared memory; V code nibbles of two
// tokens are interleaved into one byte so one table entry is a (token, token) pair at one
// dimension.  The key scale multiplies the scores, the value scale the weights, and the
// merged output is rotated back with a Walsh-Hadamard transform in registers.
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
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(src_bytes));
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
__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_f16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
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
  int b;      // global sequence
  int kvh;
  int t0;     // first token of the split (tier-relative)
  int n;      // tokens in the split
  int slot;
  int pair;   // b * Hkv + kvh: items with the same pair share their query
};

// Item order: sequence, KV head, split.  seq.item_base counts splits * Hkv per sequence.
__device__ __forceinline__ Item item_at(const AttendParams& p, int item) {
  const int bl = find_seq(p.seq, item);
  const int r = item - p.seq.item_base[bl];
  const int len = p.seq.len[bl];
  const int ns = (len + p.split_tokens - 1) / p.split_tokens;
  Item it;
  it.kvh = r / ns;
  const int split = r - it.kvh * ns;
  it.b = p.seq.b0 + bl;
  it.t0 = split * p.split_tokens;
  it.n = min(p.split_tokens, len - it.t0);
  it.slot = p.seq.slot_base[bl] + split;
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
__device__ __forceinline__ void cursor_settle(const AttendParams& p, Cursor& c, int hi, int w) {
  // move forward until the cursor sits on a step that exists
  while (c.item < hi && 16 * c.step >= c.info.n) {
    c.item += NG;
    c.step = w;
    if (c.item < hi) c.info = item_at(p, c.item);
  }
}

template <int NW, int NG>
__device__ __forceinline__ void cursor_next(const AttendParams& p, Cursor& c, int hi, int w) {
  c.step += NW;
  cursor_settle<NG>(p, c, hi, w);
}

// ------------------------------------------------------------------------------------
// online softmax of one step.  sc[j][e] (e < 2): base-2 scores of head g for tokens
// 8j + 2tq + e, masked with -inf.  Leaves the weights in sc[j][e] and returns the rescale
// factors of the accumulator columns 2tq, 2tq + 1 (column c holds head c for G = 8 and
// head c % 4 for G <= 4).  Returns false when no rescale is needed (all factors 1).
// ------------------------------------------------------------------------------------
template <int G>
__device__ __forceinline__ bool online_softmax(float (&sc)[2][4], float& m_run, float& l_run, float& a_even,
                                               float& a_odd) {
  const int lane = threadIdx.x & 31, tq = lane & 3;
  float mx = fmaxf(fmaxf(sc[0][0], sc[0][1]), fmaxf(sc[1][0], sc[1][1]));
  mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
  mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
  const float m_new = fmaxf(m_run, mx);
  const bool grow = m_new > m_run;
  const float alpha = exp2f(m_run - m_new);  // 0 on a chain's first step (m_run = -inf)
  float s = 0.f;
#pragma unroll
  for (int j = 0; j < 2; ++j)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      sc[j][e] = exp2f(sc[j][e] - m_new);
      s += sc[j][e];
    }
  l_run = l_run * alpha + s;
  m_run = m_new;
  if (!__any_sync(kFull, grow)) return false;
  constexpr int HM = G <= 4 ? 3 : 7;
  a_even = __shfl_sync(kFull, alpha, ((2 * tq) & HM) * 4);
  a_odd = __shfl_sync(kFull, alpha, ((2 * tq + 1) & HM) * 4);
  return true;
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

// Unnormalised Walsh-Hadamard transform of a 32*P-vector held P per lane (lane l holds
// elements [P*l, P*l + P)), Sylvester order.
template <int P>
__device__ __forceinline__ void warp_fwht(float (&x)[P]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int h = 1; h < P; h <<= 1)
#pragma unroll
    for (int j = 0; j < P; ++j)
      if ((j & h) == 0) {
        const float a = x[j], b = x[j + h];
        x[j] = a + b;
        x[j + h] = a - b;
      }
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    const bool upper = (lane & m) != 0;
#pragma unroll
    for (int j = 0; j < P; ++j) {
      const float o = __shfl_xor_sync(kFull, x[j], m);
      x[j] = upper ? o - x[j] : x[j] + o;
    }
  }
}

// Merge the NW chain states of a finished item (group threads) and write its partials.
// kRotate: the merged rows are in the rotated basis; rotate back (x H / D) per head.
template <int D, int G, int NW, bool kRotate>
__device__ __forceinline__ void merge_item(const AttendParams& p, const Item& it, int gi, float* area, float* mws,
                                           float* lws, float* stage) {
  const int tg = threadIdx.x - gi * NW * 32;  // thread index within the group
  const int warp_in = tg >> 5, lane = threadIdx.x & 31;
  for (int i = tg; i < G * D; i += NW * 32) {
    const int h = i / D, dim = i % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, mws[w * G + h]);
    float o = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) o = fmaf(area[(w * G + h) * D + dim], exp2f(mws[w * G + h] - M), o);
    if constexpr (kRotate) {
      stage[i] = o;
    } else {
      float L = 0.f;
#pragma unroll
      for (int w = 0; w < NW; ++w) L = fmaf(lws[w * G + h], exp2f(mws[w * G + h] - M), L);
      const int hq = it.kvh * G + h;
      p.o_part[((size_t)it.slot * p.Hq + hq) * D + dim] = o / L;
      if (dim == 0) p.lse_part[(size_t)it.slot * p.Hq + hq] = kLn2 * (M + log2f(L));
    }
  }
  if constexpr (kRotate) {
    group_sync<NW>(gi);
    constexpr int P = D / 32;
    for (int h = warp_in; h < G; h += NW) {
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < NW; ++w) M = fmaxf(M, mws[w * G + h]);
      float L = 0.f;
#pragma unroll
      for (int w = 0; w < NW; ++w) L = fmaf(lws[w * G + h], exp2f(mws[w * G + h] - M), L);
      float x[P];
#pragma unroll
      for (int j = 0; j < P; ++j) x[j] = stage[h * D + P * lane + j];
      warp_fwht<P>(x);
      const float sc = 1.f / ((float)D * L);
      const int hq = it.kvh * G + h;
      float* dst = p.o_part + ((size_t)it.slot * p.Hq + hq) * D + P * lane;
#pragma unroll
      for (int j = 0; j < P; ++j) dst[j] = x[j] * sc;
      if (lane == 0) p.lse_part[(size_t)it.slot * p.Hq + hq] = kLn2 * (M + log2f(L));
    }
  }
}

// ------------------------------------------------------------------------------------
// exact BF16 tier
// ------------------------------------------------------------------------------------
template <int D, int G, int NW, int NST>
struct Bf16Cfg {
  static constexpr int CH = D / 8;                 // 16-byte chunks per row
  static constexpr int TILE = 16 * D * 2;          // one 16-token K or V tile
  static constexpr int STAGE = 2 * TILE;
  static constexpr int LOADS = 16 * CH / 32;       // cp.async per lane per tile
  static constexpr int RINGS = NW * NST * STAGE;
  static constexpr int AREA = NW * G * D;          // floats
  static constexpr size_t SMEM = RINGS + (size_t)(AREA + 2 * NW * G) * 4;
};

template <int D, int G, int NW, int NST>
__global__ void __launch_bounds__(NW * 32, 1) attend_bf16_mma(const __grid_constant__ AttendParams p) {
  using C = Bf16Cfg<D, G, NW, NST>;
  constexpr int NG = 1;
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, tq = lane & 3;
  const int gi = 0, w = warp;
  float* area = reinterpret_cast<float*>(smem + C::RINGS);
  float* mws = area + C::AREA;
  float* lws = mws + NW * G;
  const uint32_t ring_s = smem_u32(smem + warp * NST * C::STAGE);

  int lo, hi;
  cta_range(p.seq.item_base[p.seq.n_seq], lo, hi);
  if (lo >= hi) return;

  // loads of one step into a stage; every row of the step lies in one page
  auto load_step = [&](const Item& it, int s, int st) {
    const int tok0 = it.t0 + 16 * s;
    const int nv = min(16, it.n - 16 * s);
    int64_t row0;
    if (p.tier.paged) {
      row0 = tier_page(p.tier, it.b, tok0 >> 4, p.err) * p.tier.s_seq + (int64_t)it.kvh * p.tier.s_head;
    } else {
      row0 = (int64_t)it.b * p.tier.s_seq + (int64_t)it.kvh * p.tier.s_head + (int64_t)tok0 * p.tier.s_tok;
    }
    const uint8_t* kb = p.tier.k + 2 * row0;
    const uint8_t* vb = p.tier.v + 2 * row0;
    const uint32_t st_s = ring_s + st * C::STAGE;
#pragma unroll
    for (int i = 0; i < C::LOADS; ++i) {
      const int idx = i * 32 + lane;
      const int r = idx / C::CH, c = idx % C::CH;
      const int64_t e = (int64_t)(r < nv ? r : 0) * p.tier.s_tok + 8 * c;
      const uint32_t off = (uint32_t)(r * D * 2 + ((c ^ (r & 7)) << 4));
      const int bytes = r < nv ? 16 : 0;
      cp_async16(st_s + off, kb + 2 * e, bytes);
      cp_async16(st_s + C::TILE + off, vb + 2 * e, bytes);
    }
  };

  Cursor ld;
  ld.item = lo + gi;
  ld.step = w;
  if (ld.item < hi) ld.info = item_at(p, ld.item);
  cursor_settle<NG>(p, ld, hi, w);
#pragma unroll
  for (int j = 0; j < NST; ++j) {
    if (ld.item < hi) {
      load_step(ld.info, ld.step, j);
      cursor_next<NW, NG>(p, ld, hi, w);
    }
    cp_async_commit();
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

  for (int item = lo + gi; item < hi; item += NG) {
    const Item it = item_at(p, item);
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
      cp_async_wait<NST - 1>();
      __syncwarp();
      const int nv = min(16, it.n - 16 * s);
      const uint32_t kt = ring_s + stage * C::STAGE, vt = kt + C::TILE;
      float sc[2][4];
#pragma unroll
      for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) sc[j][e] = 0.f;
#pragma unroll
      for (int kc = 0; kc < D / 16; ++kc) {
        const int mi = lane >> 3, r = (mi >> 1) * 8 + (lane & 7), c = 2 * kc + (mi & 1);
        uint32_t b[4];
        ldsm_x4(b, kt + r * D * 2 + ((c ^ (r & 7)) << 4));
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
        ldsm_x4_t(a, vt + r * D * 2 + ((c ^ (r & 7)) << 4));
        mma_bf16(acc[mt], a, pb[0], pb[1]);
        if constexpr (G > 4) mma_bf16(acc[mt], a, pl[0], pl[1]);
      }
      __syncwarp();
      if (ld.item < hi) {
        load_step(ld.info, ld.step, stage);
        cursor_next<NW, NG>(p, ld, hi, w);
      }
      cp_async_commit();
      stage = stage + 1 == NST ? 0 : stage + 1;
    }
    chain_to_smem<D, G>(acc, m_run, l_run, area + w * G * D, mws + w * G, lws + w * G, dim_of);
    group_sync<NW>(gi);
    merge_item<D, G, NW, false>(p, it, gi, area, mws, lws, nullptr);
    group_sync<NW>(gi);
  }
  cp_async_wait<0>();
}

// ------------------------------------------------------------------------------------
// compact tier (CODES4)
// ------------------------------------------------------------------------------------
// Shared memory: the lookup table lut[256][32] (entry b for lane l: the half pair
// (c[b & 15], c[b >> 4]); one copy per lane keeps the gathers conflict-free), then per
// group: the query words qw[G][D] (FP16 high/residual pairs of H q / 2^e), qscale[8],
// the merge area and staging rows; then one ring per warp.  A stage holds one 16-token
// block of K (code rows unpadded, then 16 scales) and of V (code rows padded to VROW
// bytes so the four token lanes' reads fall in different banks, then 16 scales).
template <int D, int G, int NW, int NG, int NST>
struct CodesCfg {
  static constexpr int ROWB = D / 2;
  static constexpr int VROW = ROWB + 16;
  static constexpr int K_OFF = 0;
  static constexpr int KS_OFF = 16 * ROWB;
  static constexpr int V_OFF = KS_OFF + 32;
  static constexpr int VS_OFF = V_OFF + 16 * VROW;
  static constexpr int STAGE = VS_OFF + 32;
  static constexpr int BLOCK = AKV_CODES4_BLOCK_BYTES(D);
  static constexpr int CHUNKS = BLOCK / 16;
  static constexpr int LUT = 256 * 32 * 4;
  // per-group floats: query words G*D, qscale 8, merge area NW*G*D, m and l 2*NW*G, stage G*D
  static constexpr int GROUP = G * D + 8 + NW * G * D + 2 * NW * G + G * D;
  static constexpr int RING_OFF = LUT + NG * GROUP * 4;
  static constexpr size_t SMEM = (size_t)RING_OFF + (size_t)NG * NW * NST * STAGE;
};

template <int D, int G, int NW, int NG, int NST>
__global__ void __launch_bounds__(NW * NG * 32, 1) attend_codes_mma(const __grid_constant__ AttendParams p) {
  using C = CodesCfg<D, G, NW, NG, NST>;
  constexpr int DPT = D / 8;                      // value dims per lane group
  constexpr int KB = D / 8;                       // key code bytes per lane
  constexpr int NWD = DPT / 8 > 0 ? DPT / 8 : 1;  // value code words per token per lane
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, tq = lane & 3;
  const int gi = warp / NW, w = warp % NW;
  uint32_t* lut = reinterpret_cast<uint32_t*>(smem);
  float* gbase = reinterpret_cast<float*>(smem + C::LUT) + gi * C::GROUP;
  uint32_t* qwords = reinterpret_cast<uint32_t*>(gbase);   // [G][D]
  float* qscale = gbase + G * D;                            // [8]
  float* area = qscale + 8;                                 // [NW][G][D]
  float* mws = area + NW * G * D;
  float* lws = mws + NW * G;
  float* stagef = lws + NW * G;                             // [G][D]
  uint8_t* ring = smem + C::RING_OFF + (size_t)warp * NST * C::STAGE;
  const uint32_t ring_s = smem_u32(ring);

  for (int i = threadIdx.x; i < 256 * 32; i += NW * NG * 32) {
    const int byte = i >> 5;
    lut[i] = (uint32_t)p.centroids[byte & 15] | ((uint32_t)p.centroids[byte >> 4] << 16);
  }
  __syncthreads();

  int lo, hi;
  cta_range(p.seq.item_base[p.seq.n_seq], lo, hi);
  if (lo + gi >= hi) return;  // a group without items (no block-wide barrier follows)

  auto load_step = [&](const Item& it, int s, int st) {
    const int tok0 = it.t0 + 16 * s;
    const uint8_t* kb = codes_block<D>(p.tier, p.tier.k, it.b, it.kvh, tok0, p.err);
    const uint8_t* vb = codes_block<D>(p.tier, p.tier.v, it.b, it.kvh, tok0, p.err);
    const uint32_t st_s = ring_s + st * C::STAGE;
#pragma unroll
    for (int i0 = 0; i0 < C::CHUNKS; i0 += 32) {
      const int i = i0 + lane;
      if (i < C::CHUNKS) {
        cp_async16(st_s + C::K_OFF + 16 * i, kb + 16 * i, 16);
        uint32_t voff;
        if (i < C::ROWB) {
          const int r = i / (C::ROWB / 16), c = i % (C::ROWB / 16);
          voff = C::V_OFF + r * C::VROW + 16 * c;
        } else {
          voff = C::VS_OFF + 16 * (i - C::ROWB);
        }
        cp_async16(st_s + voff, vb + 16 * i, 16);
      }
    }
  };

  Cursor ld;
  ld.item = lo + gi;
  ld.step = w;
  ld.info = item_at(p, ld.item);
  cursor_settle<NG>(p, ld, hi, w);
#pragma unroll
  for (int j = 0; j < NST; ++j) {
    if (ld.item < hi) {
      load_step(ld.info, ld.step, j);
      cursor_next<NW, NG>(p, ld, hi, w);
    }
    cp_async_commit();
  }

  const uint32_t* my_lut = lut + lane;
  auto lookup = [&](uint32_t word, int byte) -> uint32_t {
    return my_lut[__byte_perm(word, 0, 0x4440 + byte) * 32];
  };

  int dim_of[D / 16][2];
#pragma unroll
  for (int mt = 0; mt < D / 16; ++mt) {
    dim_of[mt][0] = DPT * g + mt;
    dim_of[mt][1] = DPT * g + DPT / 2 + mt;
  }
  uint32_t qa[D / 16][4];
  float kfac = 0.f;
  int q_pair = -1;
  int stage = 0;

  for (int item = lo + gi; item < hi; item += NG) {
    const Item it = item_at(p, item);
    if (it.pair != q_pair) {
      q_pair = it.pair;
      // warp h rotates head h: H q by shuffles, a power-of-two scale to [0.5, 1), FP16 hi/lo
      constexpr int P = D / 32;
      for (int h = w; h < G; h += NW) {
        const uint16_t* qrow = p.q + ((size_t)it.b * p.Hq + (size_t)it.kvh * G + h) * D + P * lane;
        float x[P];
#pragma unroll
        for (int j = 0; j < P; ++j) x[j] = bf16_to_float(qrow[j]);
        warp_fwht<P>(x);
        float mx = 0.f;
#pragma unroll
        for (int j = 0; j < P; ++j) mx = fmaxf(mx, fabsf(x[j]));
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, off));
        int e = 0;
        if (mx > 0.f) frexpf(mx, &e);
        const float inv = ldexpf(1.f, -e);
#pragma unroll
        for (int j = 0; j < P; j += 2) {
          const float x0 = x[j] * inv, x1 = x[j + 1] * inv;
          const uint32_t hw = pack_f16(x0, x1);
          const float2 hv = unpack_f16(hw);
          // (high, residual) words of dims (P*lane + j, P*lane + j + 1)
          qwords[h * D + P * lane + j] = hw;
          qwords[h * D + P * lane + j + 1] = pack_f16(x0 - hv.x, x1 - hv.y);
        }
        if (lane == 0) qscale[h] = ldexpf(1.f, e);
      }
      group_sync<NW>(gi);
      // lane (g, tq), step kc covers dims 2*KB*tq + 4kc + {0,1,2,3}: rows g = high parts,
      // rows g + 8 = residuals
      const int h = g < G ? g : 0;
      const uint32_t* qrow = qwords + h * D + 2 * KB * tq;
#pragma unroll
      for (int kc = 0; kc < D / 16; ++kc) {
        qa[kc][0] = g < G ? qrow[4 * kc] : 0u;       // high, dims 4kc, 4kc+1
        qa[kc][1] = g < G ? qrow[4 * kc + 1] : 0u;   // residual
        qa[kc][2] = g < G ? qrow[4 * kc + 2] : 0u;   // high, dims 4kc+2, 4kc+3
        qa[kc][3] = g < G ? qrow[4 * kc + 3] : 0u;   // residual
      }
      kfac = p.scale_log2 / (float)D * qscale[h];
      group_sync<NW>(gi);
    }

    float acc[D / 16][4];
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[mt][e] = 0.f;
    float m_run = -INFINITY, l_run = 0.f;

    for (int s = w; 16 * s < it.n; s += NW) {
      cp_async_wait<NST - 1>();
      __syncwarp();
      const int nv = min(16, it.n - 16 * s);
      const uint8_t* sk = ring + stage * C::STAGE;
      // ---- S^T = (H q) K_hat^T: B fragments straight from the code bytes
      float sc[2][4];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
#pragma unroll
        for (int e = 0; e < 4; ++e) sc[j][e] = 0.f;
        uint32_t wk[KB / 4];
        const uint8_t* row = sk + C::K_OFF + (8 * j + g) * C::ROWB + KB * tq;
        if constexpr (KB == 16) {
          const uint4 v = *reinterpret_cast<const uint4*>(row);
          wk[0] = v.x; wk[1] = v.y; wk[2] = v.z; wk[3] = v.w;
        } else {
          const uint2 v = *reinterpret_cast<const uint2*>(row);
          wk[0] = v.x; wk[1] = v.y;
        }
#pragma unroll
        for (int kc = 0; kc < D / 16; ++kc) {
          const uint32_t wd = wk[kc >> 1];
          mma_f16(sc[j], qa[kc], lookup(wd, 2 * (kc & 1)), lookup(wd, 2 * (kc & 1) + 1));
        }
      }
      float ksc[2][2], vsc[2][2];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const float2 kh = unpack_f16(*reinterpret_cast<const uint32_t*>(sk + C::KS_OFF + 2 * (8 * j + 2 * tq)));
        const float2 vh = unpack_f16(*reinterpret_cast<const uint32_t*>(sk + C::VS_OFF + 2 * (8 * j + 2 * tq)));
        ksc[j][0] = kh.x; ksc[j][1] = kh.y;
        vsc[j][0] = vh.x; vsc[j][1] = vh.y;
      }
      // score of head g = high row g + residual row g + 8
#pragma unroll
      for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int e = 0; e < 2; ++e) sc[j][e] = (sc[j][e] + sc[j][e + 2]) * (kfac * ksc[j][e]);
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
      // ---- P' = P * s^V (0 for masked tokens): FP16 high part and residual
      float wts[2][2];
#pragma unroll
      for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int e = 0; e < 2; ++e) wts[j][e] = sc[j][e] * vsc[j][e];
      if (nv < 16) {
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
          for (int e = 0; e < 2; ++e)
            if (8 * j + 2 * tq + e >= nv) wts[j][e] = 0.f;
      }
      uint32_t pb[2], pl[2];
      p_fragments<G, false>(wts, pb, pl);
      // ---- O_rot^T += V_hat^T P'^T: lane (g, tq) supplies value dims [DPT g, DPT g + DPT)
      // of tokens (2tq, 2tq+1) and (2tq+8, 2tq+9); one byte = the nibbles of two tokens
      uint32_t z[2][NWD][2];
#pragma unroll
      for (int pr = 0; pr < 2; ++pr) {
        const uint8_t* r0 = sk + C::V_OFF + (8 * pr + 2 * tq) * C::VROW + (DPT / 2) * g;
        const uint8_t* r1 = r0 + C::VROW;
        uint32_t w0[NWD], w1[NWD];
        if constexpr (NWD == 2) {
          const uint2 a = *reinterpret_cast<const uint2*>(r0);
          const uint2 b = *reinterpret_cast<const uint2*>(r1);
          w0[0] = a.x; w0[1] = a.y; w1[0] = b.x; w1[1] = b.y;
        } else {
          w0[0] = *reinterpret_cast<const uint32_t*>(r0);
          w1[0] = *reinterpret_cast<const uint32_t*>(r1);
        }
#pragma unroll
        for (int wi = 0; wi < NWD; ++wi) {
          z[pr][wi][0] = (w0[wi] & 0x0F0F0F0Fu) | ((w1[wi] & 0x0F0F0F0Fu) << 4);
          z[pr][wi][1] = ((w0[wi] >> 4) & 0x0F0F0F0Fu) | (w1[wi] & 0xF0F0F0F0u);
        }
      }
      // dim offset m lives in word m / 8, byte (m % 8) / 2, parity m % 2
#pragma unroll
      for (int mt = 0; mt < D / 16; ++mt) {
        uint32_t a[4];
        const int m0 = mt, m1 = DPT / 2 + mt;
        a[0] = lookup(z[0][m0 >> 3][m0 & 1], (m0 & 7) >> 1);
        a[1] = lookup(z[0][m1 >> 3][m1 & 1], (m1 & 7) >> 1);
        a[2] = lookup(z[1][m0 >> 3][m0 & 1], (m0 & 7) >> 1);
        a[3] = lookup(z[1][m1 >> 3][m1 & 1], (m1 & 7) >> 1);
        mma_f16(acc[mt], a, pb[0], pb[1]);
        if constexpr (G > 4) mma_f16(acc[mt], a, pl[0], pl[1]);
      }
      __syncwarp();
      if (ld.item < hi) {
        load_step(ld.info, ld.step, stage);
        cursor_next<NW, NG>(p, ld, hi, w);
      }
      cp_async_commit();
      stage = stage + 1 == NST ? 0 : stage + 1;
    }
    chain_to_smem<D, G>(acc, m_run, l_run, area + w * G * D, mws + w * G, lws + w * G, dim_of);
    group_sync<NW>(gi);
    merge_item<D, G, NW, true>(p, it, gi, area, mws, lws, stagef);
    group_sync<NW>(gi);
  }
  cp_async_wait<0>();
}

int sm_count() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 1;
}

template <int D, int G>
cudaError_t launch_bf16(const AttendParams& p, int n_items, cudaStream_t s) {
  constexpr int NW = 8;
  constexpr int NST = G <= 4 ? 3 : 2;
  using C = Bf16Cfg<D, G, NW, NST>;
  auto k = attend_bf16_mma<D, G, NW, NST>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM);
  if (e != cudaSuccess) return e;
  const int sms = sm_count();
  const int grid = n_items < sms ? n_items : sms;
  k<<<grid, NW * 32, C::SMEM, s>>>(p);
  return cudaGetLastError();
}

template <int D, int G>
cudaError_t launch_codes(const AttendParams& p, int n_items, cudaStream_t s) {
  constexpr int NW = 8;
  constexpr int NG = G <= 4 ? 2 : 1;
  constexpr int NST = 4;
  using C = CodesCfg<D, G, NW, NG, NST>;
  auto k = attend_codes_mma<D, G, NW, NG, NST>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM);
  if (e != cudaSuccess) return e;
  const int sms = sm_count();
  const int want = (n_items + NG - 1) / NG;
  const int grid = want < sms ? want : sms;
  k<<<grid, NW * NG * 32, C::SMEM, s>>>(p);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_d(const AttendParams& p, int G, int kind, int n_items, cudaStream_t s) {
  if (kind == AKV_TIER_BF16) {
    switch (G) {
      case 1: return launch_bf16<D, 1>(p, n_items, s);
      case 2: return launch_bf16<D, 2>(p, n_items, s);
      case 4: return launch_bf16<D, 4>(p, n_items, s);
      default: return launch_bf16<D, 8>(p, n_items, s);
    }
  }
  switch (G) {
    case 1: return launch_codes<D, 1>(p, n_items, s);
    case 2: return launch_codes<D, 2>(p, n_items, s);
    case 4: return launch_codes<D, 4>(p, n_items, s);
    default: return launch_codes<D, 8>(p, n_items, s);
  }
}

}  // namespace

// n_items counts (split, KV head) items: seq.item_base must count splits * Hkv.
cudaError_t launch_attend_mma(const AttendParams& p, int d, int G, int kind, int n_items, cudaStream_t s) {
  return d == 128 ? launch_d<128>(p, G, kind, n_items, s) : launch_d<64>(p, G, kind, n_items, s);
}

}  // namespace akv

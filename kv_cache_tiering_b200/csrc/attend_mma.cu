// Split-KV GQA decode attention on the tensor cores (mma.sync m16n8k16, float32
// accumulate), contracting across the GQA query group.
//
// One CTA (4 warps) computes one split of one sequence for one KV head and its G query
// heads.  The split is cut into 16-token steps dealt round-robin to the warps.  Each
// warp streams its steps through a private ring of shared-memory stages filled with
// cp.async (16-byte chunks, zero-filled past the end of the split) and keeps its own
// online-softmax state; the four warp states are merged at the end.
//
// Exact BF16 tier, per step:
//   S^T (heads x 16 tokens) = q (heads x d) . K^T      A = q in registers (rows >= G are
//                                                       zero), B = K rows via ldmatrix
//   O^T (d x heads)        += V^T (d x 16 tokens) . P^T A = V via ldmatrix.trans,
//                                                       B = P straight from the S^T
//                                                       accumulator registers
// P is split into a BF16 high part and a BF16 residual (two MMAs) so the weights carry
// about 16 significant bits; one BF16 rounding of P would cost up to 2^-9 relative.
// Shared-memory tiles are XOR-swizzled in 16-byte chunks so ldmatrix is conflict-free.
//
// Compact tier, per step: the same two contractions in the rotated basis ("QuantForge V2
// Walkthrough", section 1: the query is rotated instead of the keys) with FP16 operands:
// code bytes are turned into (c[lo], c[hi]) half pairs through a per-lane replicated
// lookup table in shared memory, the key scale multiplies the scores, the value scale
// the weights, and the output is rotated back with a Walsh-Hadamard transform at the end.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "akv_internal.cuh"

namespace akv {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = 32 * kWarps;
constexpr float kLn2 = 0.693147180559945309f;

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
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
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
__device__ __forceinline__ float bf16_lo_f(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi_f(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

struct Split {
  int b, bl, kvh, t0, n, slot;
};

__device__ __forceinline__ Split get_split(const AttendParams& p) {
  Split s;
  const int item = blockIdx.x;
  s.kvh = blockIdx.y;
  s.bl = find_seq(p.seq, item);
  s.b = p.seq.b0 + s.bl;
  const int split = item - p.seq.item_base[s.bl];
  s.t0 = split * p.split_tokens;
  s.n = min(p.split_tokens, p.seq.len[s.bl] - s.t0);
  s.slot = p.seq.slot_base[s.bl] + split;
  return s;
}

// Online-softmax update of one warp for one 16-token step.  sc[j][e]: base-2 scores of
// head g (lane / 4) for tokens 8j + 2tq + e of the step, already masked (-inf).  Returns
// the rescale factors for the accumulator columns (heads 2tq, 2tq + 1) and leaves the
// weights in sc.
template <int G>
__device__ __forceinline__ void online_softmax(float (&sc)[2][4], float& m_run, float& l_run, float& a_even,
                                               float& a_odd) {
  const int lane = threadIdx.x & 31, tq = lane & 3;
  float mx = fmaxf(fmaxf(sc[0][0], sc[0][1]), fmaxf(sc[1][0], sc[1][1]));
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
  const float m_new = fmaxf(m_run, mx);
  const float alpha = exp2f(m_run - m_new);  // 0 on the first step (m_run = -inf)
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
  // accumulator column c holds head c (G = 8) or head c % 4 (G <= 4: columns 4..7 carry
  // the low parts of heads 0..3)
  constexpr int HM = G <= 4 ? 3 : 7;
  a_even = __shfl_sync(0xffffffffu, alpha, ((2 * tq) & HM) * 4);
  a_odd = __shfl_sync(0xffffffffu, alpha, ((2 * tq + 1) & HM) * 4);
}

// P^T B fragments of one step from the weights w[j][e] (head g, tokens 8j + 2tq + e),
// split into a high part and a residual in the MMA's type.  G <= 4: one fragment whose
// columns 0..3 are the high parts and 4..7 the residuals of heads 0..3 (lanes of head
// group g >= 4 take the residual of head g - 4 from lane ^ 16).  G = 8: two fragments.
template <int G, bool kBF16>
__device__ __forceinline__ void p_fragments(const float (&w)[2][2], uint32_t (&b_hi)[2], uint32_t (&b_lo)[2]) {
  const int g = (threadIdx.x & 31) >> 2;
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    uint32_t hi, lo;
    if constexpr (kBF16) {
      hi = pack_bf16(w[j][0], w[j][1]);
      lo = pack_bf16(w[j][0] - bf16_lo_f(hi), w[j][1] - bf16_hi_f(hi));
    } else {
      hi = pack_f16(w[j][0], w[j][1]);
      const __half2 h2 = *reinterpret_cast<const __half2*>(&hi);
      lo = pack_f16(w[j][0] - __low2float(h2), w[j][1] - __high2float(h2));
    }
    if constexpr (G <= 4) {
      const uint32_t partner_lo = __shfl_xor_sync(0xffffffffu, lo, 16);
      b_hi[j] = g < 4 ? hi : partner_lo;
      b_lo[j] = 0u;
    } else {
      b_hi[j] = hi;
      b_lo[j] = lo;
    }
  }
}

// Merge the per-warp states through shared memory and write the split's partials.
// red: [kWarps][G][D] floats, red_m / red_l: [kWarps][G].  acc C-fragment layout:
// acc[mt][0..3] = O^T rows (dim(mt, g), dim(mt, g+8)), columns (heads 2tq, 2tq+1).
template <int D, int G, bool kRotateBack>
__device__ __forceinline__ void merge_warps_and_store(const AttendParams& p, const Split& si, float (&acc)[D / 16][4],
                                                      float m_run, float l_run, float* red, float* red_m, float* red_l,
                                                      const int (&dim_of)[D / 16][2], float out_scale) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, tq = lane & 3;
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
  if (tq == 0 && g < G) {
    red_m[warp * G + g] = m_run;
    red_l[warp * G + g] = l_run;
  }
  if constexpr (G <= 4) {  // columns 4..7 hold the residual contributions of heads 0..3
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[mt][e] += __shfl_xor_sync(0xffffffffu, acc[mt][e], 2);
  }
#pragma unroll
  for (int mt = 0; mt < D / 16; ++mt) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int h = 2 * tq + (e & 1);
      const int dim = dim_of[mt][e >> 1];
      if (h < G) red[(warp * G + h) * D + dim] = acc[mt][e];
    }
  }
  __syncthreads();
  // merged, unnormalised output staged after the warp slices
  for (int i = threadIdx.x; i < G * D; i += kThreads) {
    const int h = i / D, dim = i % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, red_m[w * G + h]);
    float o = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float sc = exp2f(red_m[w * G + h] - M);  // 0 for a warp without tokens
      o = fmaf(red[(w * G + h) * D + dim], sc, o);
    }
    red[(kWarps * G + h) * D + dim] = o;
  }
  __syncthreads();
  if constexpr (kRotateBack) {
    // in-place Walsh-Hadamard transform of the G staged rows
    float* x = red + kWarps * G * D;
    for (int hh = 1; hh < D; hh <<= 1) {
      for (int i = threadIdx.x; i < G * D / 2; i += kThreads) {
        const int row = i / (D / 2), k = i % (D / 2);
        const int j = (k / hh) * 2 * hh + (k % hh);
        const float a = x[row * D + j], b = x[row * D + j + hh];
        x[row * D + j] = a + b;
        x[row * D + j + hh] = a - b;
      }
      __syncthreads();
    }
  }
  for (int i = threadIdx.x; i < G * D; i += kThreads) {
    const int h = i / D, dim = i % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, red_m[w * G + h]);
    float L = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) L = fmaf(red_l[w * G + h], exp2f(red_m[w * G + h] - M), L);
    const int hq = si.kvh * G + h;
    p.o_part[((size_t)si.slot * p.Hq + hq) * D + dim] = red[(kWarps * G + h) * D + dim] * (out_scale / L);
    if (dim == 0) p.lse_part[(size_t)si.slot * p.Hq + hq] = kLn2 * (M + log2f(L));
  }
}

// ------------------------------------------------------------------------------------
// exact BF16 tier
// ------------------------------------------------------------------------------------
template <int D, int G, int NST>
__global__ void __launch_bounds__(kThreads) attend_bf16_mma(const __grid_constant__ AttendParams p) {
  constexpr int CH = D / 8;                 // 16-byte chunks per row
  constexpr int TILE = 16 * D * 2;          // bytes of one 16-token K (or V) tile
  constexpr int STAGE = 2 * TILE;           // K tile then V tile
  constexpr int LOADS = 16 * CH / 32;       // cp.async per lane per tile
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, tq = lane & 3;
  const Split si = get_split(p);
  uint8_t* ring = smem + warp * NST * STAGE;
  const uint32_t ring_s = smem_u32(ring);

  // A fragments of q (rows = heads; rows >= G and rows 8..15 are zero)
  uint32_t qa[D / 16][4];
  {
    const uint16_t* qrow = p.q + ((size_t)si.b * p.Hq + (size_t)si.kvh * G + (g < G ? g : 0)) * D;
#pragma unroll
    for (int kc = 0; kc < D / 16; ++kc) {
      uint32_t lo = *reinterpret_cast<const uint32_t*>(qrow + 16 * kc + 2 * tq);
      uint32_t hi = *reinterpret_cast<const uint32_t*>(qrow + 16 * kc + 8 + 2 * tq);
      qa[kc][0] = g < G ? lo : 0u;
      qa[kc][1] = 0u;
      qa[kc][2] = g < G ? hi : 0u;
      qa[kc][3] = 0u;
    }
  }

  const int nsteps = (si.n + 15) >> 4;
  const int my_steps = warp < nsteps ? (nsteps - warp + kWarps - 1) / kWarps : 0;

  // issue the cp.async of step s into stage st
  auto load_step = [&](int s, int st) {
    const int tok0 = si.t0 + 16 * s;
    const int nv = min(16, si.n - 16 * s);
    int64_t row0;  // element offset of the step's first row; rows advance by s_tok
    if (p.tier.paged) {
      row0 = tier_page(p.tier, si.b, tok0 >> 4, p.err) * p.tier.s_seq + (int64_t)si.kvh * p.tier.s_head;
    } else {
      row0 = (int64_t)si.b * p.tier.s_seq + (int64_t)si.kvh * p.tier.s_head + (int64_t)tok0 * p.tier.s_tok;
    }
    const uint32_t st_s = ring_s + st * STAGE;
#pragma unroll
    for (int i = 0; i < LOADS; ++i) {
      const int idx = i * 32 + lane;
      const int r = idx / CH, c = idx % CH;
      const int64_t e = row0 + (int64_t)(r < nv ? r : 0) * p.tier.s_tok + 8 * c;
      const uint32_t off = (uint32_t)(r * D * 2 + ((c ^ (r & 7)) << 4));
      const int bytes = r < nv ? 16 : 0;
      cp_async16(st_s + off, p.tier.k + 2 * e, bytes);
      cp_async16(st_s + TILE + off, p.tier.v + 2 * e, bytes);
    }
  };

#pragma unroll
  for (int j = 0; j < NST; ++j) {
    if (j < my_steps) load_step(warp + kWarps * j, j);
    cp_async_commit();
  }

  float acc[D / 16][4];
#pragma unroll
  for (int mt = 0; mt < D / 16; ++mt)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[mt][e] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;

  for (int i = 0; i < my_steps; ++i) {
    cp_async_wait<NST - 1>();
    __syncwarp();
    const int st = i % NST;
    const int s = warp + kWarps * i;
    const int nv = min(16, si.n - 16 * s);
    const uint32_t kt = ring_s + st * STAGE, vt = kt + TILE;

    // ---- S^T = q K^T for the step's two 8-token halves
    float sc[2][4];
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) sc[j][e] = 0.f;
#pragma unroll
    for (int kc = 0; kc < D / 16; ++kc) {
      // matrices: (half 0, chunk 2kc), (half 0, chunk 2kc+1), (half 1, 2kc), (half 1, 2kc+1)
      const int mi = lane >> 3, r = (mi >> 1) * 8 + (lane & 7), c = 2 * kc + (mi & 1);
      uint32_t b[4];
      ldsm_x4(b, kt + r * D * 2 + ((c ^ (r & 7)) << 4));
      mma_bf16(sc[0], qa[kc], b[0], b[1]);
      mma_bf16(sc[1], qa[kc], b[2], b[3]);
    }
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int t = 8 * j + 2 * tq + e;
        sc[j][e] = t < nv ? sc[j][e] * p.scale_log2 : -INFINITY;
      }
    float a_even, a_odd;
    online_softmax<G>(sc, m_run, l_run, a_even, a_odd);
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) {
      acc[mt][0] *= a_even; acc[mt][1] *= a_odd;
      acc[mt][2] *= a_even; acc[mt][3] *= a_odd;
    }
    // ---- P^T fragments: BF16 high part and BF16 residual
    const float w[2][2] = {{sc[0][0], sc[0][1]}, {sc[1][0], sc[1][1]}};
    uint32_t pb[2], pl[2];
    p_fragments<G, true>(w, pb, pl);
    // ---- O^T += V^T P^T
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) {
      // matrices: (tokens 0-7, chunk 2mt), (tokens 0-7, chunk 2mt+1), (8-15, 2mt), (8-15, 2mt+1)
      const int mi = lane >> 3, r = (mi >> 1) * 8 + (lane & 7), c = 2 * mt + (mi & 1);
      uint32_t a[4];
      ldsm_x4_t(a, vt + r * D * 2 + ((c ^ (r & 7)) << 4));
      mma_bf16(acc[mt], a, pb[0], pb[1]);
      if constexpr (G > 4) mma_bf16(acc[mt], a, pl[0], pl[1]);
    }
    __syncwarp();
    if (i + NST < my_steps) load_step(warp + kWarps * (i + NST), st);
    cp_async_commit();
  }
  cp_async_wait<0>();
  __syncthreads();

  float* red = reinterpret_cast<float*>(smem);
  float* red_m = red + (kWarps + 1) * G * D;
  float* red_l = red_m + kWarps * G;
  int dim_of[D / 16][2];
#pragma unroll
  for (int mt = 0; mt < D / 16; ++mt) {
    dim_of[mt][0] = 16 * mt + g;
    dim_of[mt][1] = 16 * mt + 8 + g;
  }
  merge_warps_and_store<D, G, false>(p, si, acc, m_run, l_run, red, red_m, red_l, dim_of, 1.0f);
}

template <int D, int G, int NST>
cudaError_t launch_bf16(const AttendParams& p, int n_items, cudaStream_t s) {
  constexpr int STAGE = 2 * 16 * D * 2;
  constexpr size_t ring = (size_t)kWarps * NST * STAGE;
  constexpr size_t red = (size_t)((kWarps + 1) * G * D + 2 * kWarps * G) * sizeof(float);
  constexpr size_t sm = ring > red ? ring : red;
  auto k = attend_bf16_mma<D, G, NST>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  k<<<dim3(n_items, p.Hkv), kThreads, sm, s>>>(p);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_bf16_d(const AttendParams& p, int G, int n_items, cudaStream_t s) {
  constexpr int NST = 3;
  switch (G) {
    case 1: return launch_bf16<D, 1, NST>(p, n_items, s);
    case 2: return launch_bf16<D, 2, NST>(p, n_items, s);
    case 4: return launch_bf16<D, 4, NST>(p, n_items, s);
    default: return launch_bf16<D, 8, NST>(p, n_items, s);
  }
}

// ------------------------------------------------------------------------------------
// compact tier (CODES4), FP16 operands in the rotated basis
// ------------------------------------------------------------------------------------
// Shared memory: the lookup table lut[256][32] (entry b, lane l: the half pair
// (c[b & 15], c[b >> 4]); one copy per lane keeps the gathers conflict-free), the rotated
// query, then one ring per warp.  A stage holds one 16-token block of K (code rows
// unpadded, then 16 scales) and of V (code rows padded to VROW bytes so the per-token
// 8-byte reads of the four token lanes fall in different banks, then 16 scales).
template <int D>
struct CodesLayout {
  static constexpr int ROWB = D / 2;            // code bytes per token
  static constexpr int VROW = ROWB + 16;        // padded V row
  static constexpr int K_OFF = 0;
  static constexpr int KS_OFF = 16 * ROWB;
  static constexpr int V_OFF = KS_OFF + 32;
  static constexpr int VS_OFF = V_OFF + 16 * VROW;
  static constexpr int STAGE = VS_OFF + 32;     // multiple of 16
  static constexpr int BLOCK = AKV_CODES4_BLOCK_BYTES(D);
  static constexpr int CHUNKS = BLOCK / 16;     // 16-byte chunks per block
};

template <int D, int G, int NST>
__global__ void __launch_bounds__(kThreads) attend_codes_mma(const __grid_constant__ AttendParams p) {
  using L = CodesLayout<D>;
  constexpr int DPT = D / 8;                    // value dims per lane group (rows g, g + 8)
  constexpr int KB = D / 8;                     // key code bytes per lane (dims [4*KB*tq, +2*KB))
  extern __shared__ __align__(128) uint8_t smem[];
  uint32_t* lut = reinterpret_cast<uint32_t*>(smem);                  // [256][32]
  float* qr = reinterpret_cast<float*>(smem + 256 * 32 * 4);           // [G][D]
  float* qscale = qr + G * D;                                          // [G]
  uint8_t* rings = smem + 256 * 32 * 4 + (G * D + 8) * 4;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, tq = lane & 3;
  const Split si = get_split(p);
  uint8_t* ring = rings + warp * NST * L::STAGE;
  const uint32_t ring_s = smem_u32(ring);

  const int nsteps = (si.n + 15) >> 4;
  const int my_steps = warp < nsteps ? (nsteps - warp + kWarps - 1) / kWarps : 0;
  auto load_step = [&](int s, int st) {
    const int tok0 = si.t0 + 16 * s;
    const uint8_t* kb = codes_block<D>(p.tier, p.tier.k, si.b, si.kvh, tok0, p.err);
    const uint8_t* vb = codes_block<D>(p.tier, p.tier.v, si.b, si.kvh, tok0, p.err);
    const uint32_t st_s = ring_s + st * L::STAGE;
    for (int i = lane; i < L::CHUNKS; i += 32) {
      // K: rows unpadded, scales right after -- the block's own layout
      cp_async16(st_s + L::K_OFF + 16 * i, kb + 16 * i, 16);
      uint32_t voff;
      if (i < 16 * L::ROWB / 16) {
        const int r = i / (L::ROWB / 16), c = i % (L::ROWB / 16);
        voff = L::V_OFF + r * L::VROW + 16 * c;
      } else {
        voff = L::VS_OFF + 16 * (i - 16 * L::ROWB / 16);
      }
      cp_async16(st_s + voff, vb + 16 * i, 16);
    }
  };
#pragma unroll
  for (int j = 0; j < NST; ++j) {
    if (j < my_steps) load_step(warp + kWarps * j, j);
    cp_async_commit();
  }

  // lookup table and rotated query (overlaps the first loads)
  for (int i = threadIdx.x; i < 256 * 32; i += kThreads) {
    const int byte = i >> 5;
    lut[i] = (uint32_t)p.centroids[byte & 15] | ((uint32_t)p.centroids[byte >> 4] << 16);
  }
  for (int i = threadIdx.x; i < G * D; i += kThreads) {
    const int h = i / D, dd = i % D;
    qr[i] = bf16_to_float(p.q[((size_t)si.b * p.Hq + (size_t)si.kvh * G + h) * D + dd]);
  }
  __syncthreads();
  for (int hh = 1; hh < D; hh <<= 1) {
    for (int i = threadIdx.x; i < G * D / 2; i += kThreads) {
      const int row = i / (D / 2), k = i % (D / 2);
      const int j = (k / hh) * 2 * hh + (k % hh);
      const float a = qr[row * D + j], b = qr[row * D + j + hh];
      qr[row * D + j] = a + b;
      qr[row * D + j + hh] = a - b;
    }
    __syncthreads();
  }
  // per head: power-of-two scale bringing max |H q| into [0.5, 1) for FP16
  for (int h = warp; h < G; h += kWarps) {
    float mx = 0.f;
    for (int i = lane; i < D; i += 32) mx = fmaxf(mx, fabsf(qr[h * D + i]));
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    int e = 0;
    if (mx > 0.f) frexpf(mx, &e);
    if (lane == 0) qscale[h] = ldexpf(1.f, e);
  }
  __syncthreads();
  // A fragments of H q / 2^e: lane (g, tq), step kc covers dims 2*KB*tq + 4kc + {0,1,2,3}
  uint32_t qa[D / 16][4];
  float kfac = 0.f;
  {
    const int h = g < G ? g : 0;
    const float inv = 1.f / qscale[h];
    const float* row = qr + h * D + 2 * KB * tq;
    // rows g: FP16 high part of head g; rows g + 8: its FP16 residual
    auto hi_lo = [&](float x0, float x1, uint32_t& hi, uint32_t& lo) {
      hi = pack_f16(x0, x1);
      const __half2 h2 = *reinterpret_cast<const __half2*>(&hi);
      lo = pack_f16(x0 - __low2float(h2), x1 - __high2float(h2));
    };
#pragma unroll
    for (int kc = 0; kc < D / 16; ++kc) {
      uint32_t h0, l0, h1, l1;
      hi_lo(row[4 * kc] * inv, row[4 * kc + 1] * inv, h0, l0);
      hi_lo(row[4 * kc + 2] * inv, row[4 * kc + 3] * inv, h1, l1);
      qa[kc][0] = g < G ? h0 : 0u;
      qa[kc][1] = g < G ? l0 : 0u;
      qa[kc][2] = g < G ? h1 : 0u;
      qa[kc][3] = g < G ? l1 : 0u;
    }
    // base-2 score = scale_log2 / D * s_t * 2^e * (codes . H q / 2^e)
    kfac = p.scale_log2 / (float)D * qscale[h];
  }
  const uint32_t* my_lut = lut + lane;

  float acc[D / 16][4];
#pragma unroll
  for (int mt = 0; mt < D / 16; ++mt)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[mt][e] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;

  for (int i = 0; i < my_steps; ++i) {
    cp_async_wait<NST - 1>();
    __syncwarp();
    const int st = i % NST;
    const int s = warp + kWarps * i;
    const int nv = min(16, si.n - 16 * s);
    const uint8_t* sk = ring + st * L::STAGE;

    // ---- S^T = (H q) K_hat^T; B fragments straight from the code bytes
    float sc[2][4];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
#pragma unroll
      for (int e = 0; e < 4; ++e) sc[j][e] = 0.f;
      uint32_t w[KB / 4];
      const uint8_t* row = sk + L::K_OFF + (8 * j + g) * L::ROWB + KB * tq;
      if constexpr (KB == 16) {
        const uint4 v = *reinterpret_cast<const uint4*>(row);
        w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
      } else {
        const uint2 v = *reinterpret_cast<const uint2*>(row);
        w[0] = v.x; w[1] = v.y;
      }
#pragma unroll
      for (int kc = 0; kc < D / 16; ++kc) {
        const uint32_t wd = w[kc >> 1];
        const uint32_t b0 = my_lut[__byte_perm(wd, 0, 0x4440 + 2 * (kc & 1)) * 32];
        const uint32_t b1 = my_lut[__byte_perm(wd, 0, 0x4441 + 2 * (kc & 1)) * 32];
        mma_f16(sc[j], qa[kc], b0, b1);
      }
    }
    // scales of the lane's four tokens 8j + 2tq + e
    float ksc[2][2], vsc[2][2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const __half2 kh = *reinterpret_cast<const __half2*>(sk + L::KS_OFF + 2 * (8 * j + 2 * tq));
      const __half2 vh = *reinterpret_cast<const __half2*>(sk + L::VS_OFF + 2 * (8 * j + 2 * tq));
      ksc[j][0] = __low2float(kh); ksc[j][1] = __high2float(kh);
      vsc[j][0] = __low2float(vh); vsc[j][1] = __high2float(vh);
    }
    // score of head g = high row g + residual row g + 8
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int t = 8 * j + 2 * tq + e;
        sc[j][e] = t < nv ? (sc[j][e] + sc[j][e + 2]) * (kfac * ksc[j][e]) : -INFINITY;
      }
    float a_even, a_odd;
    online_softmax<G>(sc, m_run, l_run, a_even, a_odd);
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) {
      acc[mt][0] *= a_even; acc[mt][1] *= a_odd;
      acc[mt][2] *= a_even; acc[mt][3] *= a_odd;
    }
    // ---- P' = P * s^V (masked tokens 0): FP16 high part and residual
    float w[2][2];
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
      for (int e = 0; e < 2; ++e) w[j][e] = (8 * j + 2 * tq + e < nv) ? sc[j][e] * vsc[j][e] : 0.f;
    uint32_t pb[2], pl[2];
    p_fragments<G, false>(w, pb, pl);
    // ---- O_rot^T += V_hat^T P'^T: lane (g, tq) supplies value dims [DPT*g, DPT*g + DPT)
    // of tokens (2tq, 2tq+1) and (2tq+8, 2tq+9); nibbles of two tokens at the same dim
    // are interleaved into one byte, whose table entry is the (token, token) half pair.
    uint32_t z[2][DPT / 8 > 0 ? DPT / 8 : 1][2];  // [token pair][word][even/odd dims]
#pragma unroll
    for (int pr = 0; pr < 2; ++pr) {
      const int t0 = 8 * pr + 2 * tq;
      const uint8_t* r0 = sk + L::V_OFF + t0 * L::VROW + (DPT / 2) * g;
      const uint8_t* r1 = r0 + L::VROW;
      uint32_t w0[DPT / 8 > 0 ? DPT / 8 : 1], w1[DPT / 8 > 0 ? DPT / 8 : 1];
      if constexpr (DPT == 16) {
        const uint2 a = *reinterpret_cast<const uint2*>(r0);
        const uint2 b = *reinterpret_cast<const uint2*>(r1);
        w0[0] = a.x; w0[1] = a.y; w1[0] = b.x; w1[1] = b.y;
      } else {
        w0[0] = *reinterpret_cast<const uint32_t*>(r0);
        w1[0] = *reinterpret_cast<const uint32_t*>(r1);
      }
#pragma unroll
      for (int wi = 0; wi < (DPT / 8 > 0 ? DPT / 8 : 1); ++wi) {
        z[pr][wi][0] = (w0[wi] & 0x0F0F0F0Fu) | ((w1[wi] & 0x0F0F0F0Fu) << 4);
        z[pr][wi][1] = ((w0[wi] >> 4) & 0x0F0F0F0Fu) | (w1[wi] & 0xF0F0F0F0u);
      }
    }
    // dim offset m (0 <= m < DPT) lives in word m / 8, byte (m % 8) / 2, parity m % 2
    auto vlookup = [&](int pr, int m) -> uint32_t {
      const uint32_t zz = z[pr][m >> 3][m & 1];
      return my_lut[__byte_perm(zz, 0, 0x4440 + ((m & 7) >> 1)) * 32];
    };
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) {
      uint32_t a[4];
      a[0] = vlookup(0, mt);              // row g,     tokens 2tq, 2tq+1
      a[1] = vlookup(0, DPT / 2 + mt);    // row g + 8, tokens 2tq, 2tq+1
      a[2] = vlookup(1, mt);              // row g,     tokens 2tq+8, 2tq+9
      a[3] = vlookup(1, DPT / 2 + mt);    // row g + 8
      mma_f16(acc[mt], a, pb[0], pb[1]);
      if constexpr (G > 4) mma_f16(acc[mt], a, pl[0], pl[1]);
    }
    __syncwarp();
    if (i + NST < my_steps) load_step(warp + kWarps * (i + NST), st);
    cp_async_commit();
  }
  cp_async_wait<0>();
  __syncthreads();

  float* red = reinterpret_cast<float*>(smem);
  float* red_m = red + (kWarps + 1) * G * D;
  float* red_l = red_m + kWarps * G;
  int dim_of[D / 16][2];
#pragma unroll
  for (int mt = 0; mt < D / 16; ++mt) {
    dim_of[mt][0] = DPT * g + mt;
    dim_of[mt][1] = DPT * g + DPT / 2 + mt;
  }
  // O = H (sum_t p_t s^V_t c[code_t]) / (D l)
  merge_warps_and_store<D, G, true>(p, si, acc, m_run, l_run, red, red_m, red_l, dim_of, 1.0f / (float)D);
}

template <int D, int G, int NST>
cudaError_t launch_codes(const AttendParams& p, int n_items, cudaStream_t s) {
  using L = CodesLayout<D>;
  constexpr size_t head = (size_t)256 * 32 * 4 + (size_t)(G * D + 8) * 4;
  constexpr size_t rings = (size_t)kWarps * NST * L::STAGE;
  constexpr size_t red = (size_t)((kWarps + 1) * G * D + 2 * kWarps * G) * sizeof(float);
  constexpr size_t sm = (head + rings) > red ? (head + rings) : red;
  auto k = attend_codes_mma<D, G, NST>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  k<<<dim3(n_items, p.Hkv), kThreads, sm, s>>>(p);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_codes_d(const AttendParams& p, int G, int n_items, cudaStream_t s) {
  constexpr int NST = 6;
  switch (G) {
    case 1: return launch_codes<D, 1, NST>(p, n_items, s);
    case 2: return launch_codes<D, 2, NST>(p, n_items, s);
    case 4: return launch_codes<D, 4, NST>(p, n_items, s);
    default: return launch_codes<D, 8, NST>(p, n_items, s);
  }
}

}  // namespace

cudaError_t launch_attend_mma(const AttendParams& p, int d, int G, int kind, int n_items, cudaStream_t s) {
  if (kind == AKV_TIER_BF16)
    return d == 128 ? launch_bf16_d<128>(p, G, n_items, s) : launch_bf16_d<64>(p, G, n_items, s);
  return d == 128 ? launch_codes_d<128>(p, G, n_items, s) : launch_codes_d<64>(p, G, n_items, s);
}

}  // namespace akv

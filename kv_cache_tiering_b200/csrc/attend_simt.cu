// Split-KV GQA decode attention on CUDA cores (float32 FMA), exact BF16 tier and compact
// tier.  One CTA (256 threads) computes one split of one sequence for one KV head and
// all G query heads that read it, in three phases:
//   A  scores: half-warps (d/8 lanes, 16 bytes each) stream the split's key rows with
//      coalesced 16-byte loads; partial dot products for the G heads are reduced by a
//      transposing butterfly that leaves each lane one head's score;
//   B  softmax statistics per head over the split (max, exp2, sum) in shared memory;
//   C  values: each warp owns 32 dimensions and 8 token lanes; weights come from shared
//      memory, partial sums are reduced across lanes and warps at the end.
// K and V are each read from HBM exactly once.  Scores are kept in base-2 units
// (softmax_scale * log2 e folded into q), so LSE = ln 2 * (m + log2 l).
//
// The compact tier runs the same phases in the rotated basis ("QuantForge V2
// Walkthrough", section 1: rotate the query, not the keys): q is rotated once per CTA
// by an in-shared-memory Walsh-Hadamard transform, codes are dequantised through a
// byte -> (c[lo], c[hi]) table in shared memory, the per-token scales are applied to
// the scores and the weights, and the output is rotated back at the end.
#include <cuda_fp16.h>

#include "akv_internal.cuh"

namespace akv {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr float kLn2 = 0.693147180559945309f;

// Reduce vals[0..G) over the LPT lanes of a lane group (LPT a power of two, G <= LPT).
// Each halving step sends half of the remaining heads to the partner and keeps the other
// half, so the exchange costs G-1 + log2(LPT/G) shuffles.  On return vals[0] holds the
// full sum of head head_of_lane(lane).
template <int G, int LPT>
__device__ __forceinline__ void group_reduce(float (&vals)[G], int lane) {
  int cnt = G;
#pragma unroll
  for (int off = LPT / 2; off >= 1; off >>= 1) {
    if (cnt > 1) {
      const bool upper = (lane & off) != 0;
#pragma unroll
      for (int j = 0; j < G / 2; ++j) {
        if (j < cnt / 2) {
          float send = upper ? vals[j] : vals[j + cnt / 2];
          float keep = upper ? vals[j + cnt / 2] : vals[j];
          vals[j] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
      }
      cnt >>= 1;
    } else {
      vals[0] += __shfl_xor_sync(0xffffffffu, vals[0], off);
    }
  }
}

template <int G, int LPT>
__device__ __forceinline__ int head_of_lane(int lane) {
  int h = 0, cnt = G;
  for (int off = LPT / 2; off >= 1 && cnt > 1; off >>= 1) {
    cnt >>= 1;
    if (lane & off) h += cnt;
  }
  return h;
}

struct SplitInfo {
  int b;        // global sequence index
  int bl;       // launch-local
  int kvh;
  int t0;       // first token of the split (tier-relative)
  int n;        // tokens in the split
  int slot;
};

__device__ __forceinline__ SplitInfo split_info(const AttendParams& p) {
  SplitInfo s;
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

// Phase B: per-head max / exp2 / sum over sc[t*G + h], t < n.  Writes p in place.
template <int G>
__device__ __forceinline__ void softmax_stats(float* sc, int n, float* sm_m, float* sm_l) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int h = warp; h < G; h += kWarps) {
    float m = -INFINITY;
    for (int t = lane; t < n; t += 32) m = fmaxf(m, sc[t * G + h]);
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    float l = 0.f;
    for (int t = lane; t < n; t += 32) {
      float e = exp2f(sc[t * G + h] - m);
      sc[t * G + h] = e;
      l += e;
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
    if (lane == 0) { sm_m[h] = m; sm_l[h] = l; }
  }
}

// Load the G weights of token t from sc[t*G ...].
template <int G>
__device__ __forceinline__ void load_weights(const float* sc, int t, float (&w)[G]) {
  if constexpr (G == 1) {
    w[0] = sc[t];
  } else if constexpr (G == 2) {
    float2 a = *reinterpret_cast<const float2*>(sc + 2 * t); w[0] = a.x; w[1] = a.y;
  } else {
#pragma unroll
    for (int j = 0; j < G; j += 4) {
      float4 a = *reinterpret_cast<const float4*>(sc + G * t + j);
      w[j] = a.x; w[j + 1] = a.y; w[j + 2] = a.z; w[j + 3] = a.w;
    }
  }
}

// Phase C epilogue: reduce acc[G][8] over the 8 token lanes of the warp and over the
// token phases, into red[G][D] (sum of all phases).  Lane layout: tsub = lane >> 2,
// dch = lane & 3, dims [32*dg + 8*dch, +8).
template <int D, int G>
__device__ __forceinline__ void reduce_pv(float (&acc)[G][8], float* red, int dg, int ph) {
  constexpr int DG = D / 32, TPH = kWarps / DG;
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float v = acc[h][i];
      v += __shfl_xor_sync(0xffffffffu, v, 4);
      v += __shfl_xor_sync(0xffffffffu, v, 8);
      v += __shfl_xor_sync(0xffffffffu, v, 16);
      acc[h][i] = v;
    }
  // phases write in turn (ph = 0 first) so the sum order is fixed
  const int dbase = 32 * dg + 8 * (lane & 3);
  for (int r = 0; r < TPH; ++r) {
    if (ph == r && lane < 4) {
#pragma unroll
      for (int h = 0; h < G; ++h)
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          float* dst = red + h * D + dbase + i;
          *dst = (r == 0) ? acc[h][i] : (*dst + acc[h][i]);
        }
    }
    __syncthreads();
  }
}

// In-place unnormalised Walsh-Hadamard transform of G rows of D floats in shared memory.
template <int D, int G>
__device__ __forceinline__ void smem_fwht(float* x) {
  for (int h = 1; h < D; h <<= 1) {
    for (int i = threadIdx.x; i < G * D / 2; i += kThreads) {
      const int row = i / (D / 2), k = i % (D / 2);
      const int j = (k / h) * 2 * h + (k % h);
      float a = x[row * D + j], b = x[row * D + j + h];
      x[row * D + j] = a + b;
      x[row * D + j + h] = a - b;
    }
    __syncthreads();
  }
}

// ------------------------------------------------------------------------------------
// exact BF16 tier
// ------------------------------------------------------------------------------------
template <int D, int G>
__global__ void __launch_bounds__(kThreads) attend_bf16_simt(const __grid_constant__ AttendParams p) {
  constexpr int LPT = D / 8;        // lanes per token row (16 bytes each)
  constexpr int TPR = 32 / LPT;     // token rows per warp pass
  constexpr int DG = D / 32, TPH = kWarps / DG;
  extern __shared__ float smem[];
  float* sc = smem;                              // [split_tokens][G]
  float* red = sc + p.split_tokens * G;          // [G][D]
  __shared__ float sm_m[G], sm_l[G];

  const SplitInfo si = split_info(p);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint8_t* kbase = p.tier.k;
  const uint8_t* vbase = p.tier.v;

  // ---- phase A: scores
  {
    const int tsub = lane / LPT, ch = lane % LPT;
    float qf[G][8];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const uint16_t* qrow = p.q + ((size_t)si.b * p.Hq + (size_t)si.kvh * G + h) * D + 8 * ch;
      uint4 w = *reinterpret_cast<const uint4*>(qrow);
      qf[h][0] = bf16lo(w.x) * p.scale_log2; qf[h][1] = bf16hi(w.x) * p.scale_log2;
      qf[h][2] = bf16lo(w.y) * p.scale_log2; qf[h][3] = bf16hi(w.y) * p.scale_log2;
      qf[h][4] = bf16lo(w.z) * p.scale_log2; qf[h][5] = bf16hi(w.z) * p.scale_log2;
      qf[h][6] = bf16lo(w.w) * p.scale_log2; qf[h][7] = bf16hi(w.w) * p.scale_log2;
    }
    const int my_head = head_of_lane<G, LPT>(lane % LPT);
    const bool writer = ((lane % LPT) & (LPT / G - 1)) == 0;
    constexpr int U = 4;
    for (int base = warp * TPR; base < si.n; base += kWarps * TPR * U) {
      uint4 kw[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int tt = base + u * kWarps * TPR + tsub;
        if (tt < si.n) kw[u] = *reinterpret_cast<const uint4*>(bf16_row(p.tier, kbase, si.b, si.kvh, si.t0 + tt, p.err) + 16 * ch);
        else kw[u] = make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int tt = base + u * kWarps * TPR + tsub;
        float k8[8] = {bf16lo(kw[u].x), bf16hi(kw[u].x), bf16lo(kw[u].y), bf16hi(kw[u].y),
                       bf16lo(kw[u].z), bf16hi(kw[u].z), bf16lo(kw[u].w), bf16hi(kw[u].w)};
        float part[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
          float a = 0.f;
#pragma unroll
          for (int i = 0; i < 8; ++i) a = fmaf(qf[h][i], k8[i], a);
          part[h] = a;
        }
        group_reduce<G, LPT>(part, lane % LPT);
        if (writer && tt < si.n) sc[tt * G + my_head] = part[0];
      }
    }
  }
  __syncthreads();
  softmax_stats<G>(sc, si.n, sm_m, sm_l);
  __syncthreads();

  // ---- phase C: values
  {
    const int dg = warp % DG, ph = warp / DG;
    const int tsub = lane >> 2, dch = lane & 3;
    float acc[G][8];
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[h][i] = 0.f;
    constexpr int STRIDE = TPH * 8;
    constexpr int U = 4;
    const int col = 32 * dg + 8 * dch;
    for (int base = ph * 8 + tsub; base < si.n; base += STRIDE * U) {
      uint4 vw[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int tt = base + u * STRIDE;
        if (tt < si.n) vw[u] = *reinterpret_cast<const uint4*>(bf16_row(p.tier, vbase, si.b, si.kvh, si.t0 + tt, p.err) + 2 * col);
        else vw[u] = make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int tt = base + u * STRIDE;
        if (tt < si.n) {
          float w[G];
          load_weights<G>(sc, tt, w);
          float v8[8] = {bf16lo(vw[u].x), bf16hi(vw[u].x), bf16lo(vw[u].y), bf16hi(vw[u].y),
                         bf16lo(vw[u].z), bf16hi(vw[u].z), bf16lo(vw[u].w), bf16hi(vw[u].w)};
#pragma unroll
          for (int h = 0; h < G; ++h)
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[h][i] = fmaf(w[h], v8[i], acc[h][i]);
        }
      }
    }
    reduce_pv<D, G>(acc, red, dg, ph);
  }

  // ---- epilogue
  for (int i = threadIdx.x; i < G * D; i += kThreads) {
    const int h = i / D, dd = i % D;
    const int hq = si.kvh * G + h;
    p.o_part[((size_t)si.slot * p.Hq + hq) * D + dd] = red[i] / sm_l[h];
  }
  if (threadIdx.x < G) {
    const int h = threadIdx.x;
    p.lse_part[(size_t)si.slot * p.Hq + si.kvh * G + h] = kLn2 * (sm_m[h] + log2f(sm_l[h]));
  }
}

// ------------------------------------------------------------------------------------
// compact tier (CODES4)
// ------------------------------------------------------------------------------------
// Value codes of dims col .. col + 7 (col a multiple of 8) of token t of a value block, in
// the key row layout (byte j = dims col + 2j, col + 2j + 1).  A value block stores token
// pairs: byte k of pair row r holds dim k of tokens 2r and 2r + 1, units of D/8 bytes at
// position u ^ w(r).
template <int D>
__device__ __forceinline__ uint32_t value_codes8(const uint8_t* blk, int t, int col) {
  constexpr int US = D / 8;
  const int r = t >> 1;
  const int w = D == 128 ? 2 * (r & 3) : 4 * ((r >> 1) & 1);
  const uint2 v = *reinterpret_cast<const uint2*>(blk + r * D + ((col / US) ^ w) * US + col % US);
  const int sh = 4 * (t & 1);
  uint32_t x = (v.x >> sh) & 0x0F0F0F0Fu, y = (v.y >> sh) & 0x0F0F0F0Fu;
  x |= x >> 4;  // bytes 0 and 2 now hold dim pairs (0, 1) and (2, 3)
  y |= y >> 4;
  return __byte_perm(x, y, 0x6420);
}

template <int D, int G>
__global__ void __launch_bounds__(kThreads) attend_codes_simt(const __grid_constant__ AttendParams p) {
  constexpr int LPT = D / 8;        // lanes per token: 8 coordinates = 4 code bytes each
  constexpr int TPR = 32 / LPT;
  constexpr int DG = D / 32, TPH = kWarps / DG;
  constexpr int ROWB = D / 2;       // code bytes per token row
  extern __shared__ float smem[];
  float* sc = smem;                              // [split_tokens][G]
  float* red = sc + p.split_tokens * G;          // [G][D]
  float* qr = red + G * D;                       // [G][D] rotated query
  __shared__ float2 lut[256];
  __shared__ float sm_m[G], sm_l[G];

  const SplitInfo si = split_info(p);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  for (int i = threadIdx.x; i < 256; i += kThreads)
    lut[i] = make_float2(half_bits_to_float(p.centroids[i & 15]), half_bits_to_float(p.centroids[i >> 4]));
  for (int i = threadIdx.x; i < G * D; i += kThreads) {
    const int h = i / D, dd = i % D;
    qr[i] = bf16_to_float(p.q[((size_t)si.b * p.Hq + (size_t)si.kvh * G + h) * D + dd]) * coord_sign(p.tier, dd);
  }
  __syncthreads();
  smem_fwht<D, G>(qr);  // qr = H (s . q) (unnormalised); ends with __syncthreads

  // score_t (base 2) = scale_log2 * s_t / D * (H q) . c[codes_t]
  const float kfac = p.scale_log2 / (float)D;

  // ---- phase A
  {
    const int tsub = lane / LPT, ch = lane % LPT;
    float qf[G][8];
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int i = 0; i < 8; ++i) qf[h][i] = qr[h * D + 8 * ch + i] * kfac;
    const int my_head = head_of_lane<G, LPT>(lane % LPT);
    const bool writer = ((lane % LPT) & (LPT / G - 1)) == 0;
    constexpr int U = 4;
    for (int base = warp * TPR; base < si.n; base += kWarps * TPR * U) {
      uint32_t cw[U];
      float sk[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int tt = base + u * kWarps * TPR + tsub;
        if (tt < si.n) {
          const int tok = si.t0 + tt;
          const uint8_t* blk = codes_block<D>(p.tier, p.tier.k, si.b, si.kvh, tok, p.err);
          cw[u] = *reinterpret_cast<const uint32_t*>(blk + (tok & 15) * ROWB + 4 * ch);
          sk[u] = half_bits_to_float(*reinterpret_cast<const uint16_t*>(blk + 16 * ROWB + 2 * (tok & 15)));
        } else {
          cw[u] = 0x77777777u;
          sk[u] = 0.f;
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int tt = base + u * kWarps * TPR + tsub;
        float k8[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float2 c2 = lut[(cw[u] >> (8 * j)) & 0xff];
          k8[2 * j] = c2.x; k8[2 * j + 1] = c2.y;
        }
        float part[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
          float a = 0.f;
#pragma unroll
          for (int i = 0; i < 8; ++i) a = fmaf(qf[h][i], k8[i], a);
          part[h] = a;
        }
        group_reduce<G, LPT>(part, lane % LPT);
        if (writer && tt < si.n) sc[tt * G + my_head] = part[0] * sk[u];
      }
    }
  }
  __syncthreads();
  softmax_stats<G>(sc, si.n, sm_m, sm_l);
  __syncthreads();

  // ---- phase C: rotated-basis values, weights scaled by the value scale s^V_t
  {
    const int dg = warp % DG, ph = warp / DG;
    const int tsub = lane >> 2, dch = lane & 3;
    float acc[G][8];
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[h][i] = 0.f;
    constexpr int STRIDE = TPH * 8;
    constexpr int U = 4;
    const int col = 32 * dg + 8 * dch;
    for (int base = ph * 8 + tsub; base < si.n; base += STRIDE * U) {
      uint32_t cw[U];
      float sv[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int tt = base + u * STRIDE;
        if (tt < si.n) {
          const int tok = si.t0 + tt;
          const uint8_t* blk = codes_block<D>(p.tier, p.tier.v, si.b, si.kvh, tok, p.err);
          cw[u] = value_codes8<D>(blk, tok & 15, col);
          sv[u] = half_bits_to_float(*reinterpret_cast<const uint16_t*>(blk + 16 * ROWB + 2 * (tok & 15)));
        } else {
          cw[u] = 0x77777777u;
          sv[u] = 0.f;
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int tt = base + u * STRIDE;
        if (tt < si.n) {
          float w[G];
          load_weights<G>(sc, tt, w);
          float v8[8];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            float2 c2 = lut[(cw[u] >> (8 * j)) & 0xff];
            v8[2 * j] = c2.x; v8[2 * j + 1] = c2.y;
          }
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const float wh = w[h] * sv[u];
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[h][i] = fmaf(wh, v8[i], acc[h][i]);
          }
        }
      }
    }
    reduce_pv<D, G>(acc, red, dg, ph);
  }
  // rotate back: O = s . (H acc) / (D * l)
  smem_fwht<D, G>(red);
  for (int i = threadIdx.x; i < G * D; i += kThreads) {
    const int h = i / D, dd = i % D;
    const int hq = si.kvh * G + h;
    p.o_part[((size_t)si.slot * p.Hq + hq) * D + dd] = red[i] * coord_sign(p.tier, dd) / ((float)D * sm_l[h]);
  }
  if (threadIdx.x < G) {
    const int h = threadIdx.x;
    p.lse_part[(size_t)si.slot * p.Hq + si.kvh * G + h] = kLn2 * (sm_m[h] + log2f(sm_l[h]));
  }
}

template <int D, int G>
cudaError_t launch_simt_dg(const AttendParams& p, int kind, int n_items, cudaStream_t s) {
  dim3 grid(n_items, p.Hkv);
  if (kind == AKV_TIER_BF16) {
    const size_t sm = (size_t)(p.split_tokens * G + G * D) * sizeof(float);
    auto k = attend_bf16_simt<D, G>;
    cudaError_t e = ensure_smem<attend_bf16_simt<D, G>>((int)sm);
    if (e != cudaSuccess) return e;
    k<<<grid, kThreads, sm, s>>>(p);
  } else {
    const size_t sm = (size_t)(p.split_tokens * G + 2 * G * D) * sizeof(float);
    auto k = attend_codes_simt<D, G>;
    cudaError_t e = ensure_smem<attend_codes_simt<D, G>>((int)sm);
    if (e != cudaSuccess) return e;
    k<<<grid, kThreads, sm, s>>>(p);
  }
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_simt_d(const AttendParams& p, int G, int kind, int n_items, cudaStream_t s) {
  switch (G) {
    case 1: return launch_simt_dg<D, 1>(p, kind, n_items, s);
    case 2: return launch_simt_dg<D, 2>(p, kind, n_items, s);
    case 4: return launch_simt_dg<D, 4>(p, kind, n_items, s);
    default: return launch_simt_dg<D, 8>(p, kind, n_items, s);
  }
}

}  // namespace

cudaError_t launch_attend_simt(const AttendParams& p, int d, int G, int kind, int n_items, cudaStream_t s) {
  return d == 128 ? launch_simt_d<128>(p, G, kind, n_items, s) : launch_simt_d<64>(p, G, kind, n_items, s);
}

}  // namespace akv

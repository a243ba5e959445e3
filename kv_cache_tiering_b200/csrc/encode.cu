// Compact-tier encoder: Walsh-Hadamard rotation, binary16 L2-norm scale, 4-bit Lloyd-Max
// codes, nibble packing into 16-token blocks (the compact form of the hybrid tier of
// "Context beyond VRAM", section "What I built"; rotation before quantisation as in
// "QuantForge V2 Walkthrough", section 1).
//
// One warp encodes one (token, KV head) vector; a CTA of 16 warps covers one 16-token
// block of one KV head, K and V.  Arithmetic is float64 and follows the definition
// step for step, so codes and scales are bit-exact against a float64 reference:
//   * lane l holds coordinates [P*l, P*l + P), P = D/32;
//   * butterfly stage h maps (z_j, z_{j+h}) to (z_j + z_{j+h}, z_j - z_{j+h}); stages
//     with h < P run inside a lane, the others exchange with lane l ^ (h / P);
//   * the sum of squares is the pairwise-halving sum: inside the lane first, then a
//     butterfly over lanes with masks 1, 2, 4, 8, 16 (IEEE addition commutes, so every
//     lane ends with the same value, equal to the pairwise tree);
//   * s = binary16(sqrt(ss)) with one rounding from float64 (cvt.rn.f16.f64);
//   * code = number of boundaries b_j with z > s * b_j (each product exact in float64).
#include <cuda_fp16.h>

#include "akv_internal.cuh"

namespace akv {
namespace {

// Encode one vector: its code row (D/2 bytes, code 2k in the low nibble of byte k) goes to
// code_row, its binary16 scale to scale_slot.
template <int D>
__device__ __forceinline__ void encode_vector(const uint8_t* src_row, uint8_t* code_row, uint16_t* scale_slot,
                                              bool valid, const double* bound, const uint32_t* signs, int32_t* err) {
  constexpr int P = D / 32;  // coordinates per lane: 4 (d = 128) or 2 (d = 64)
  const int lane = threadIdx.x & 31;
  double z[P];
  bool finite = true;
  if (valid) {
    if constexpr (P == 4) {
      uint2 w = *reinterpret_cast<const uint2*>(src_row + 8 * lane);
      z[0] = (double)bf16lo(w.x); z[1] = (double)bf16hi(w.x);
      z[2] = (double)bf16lo(w.y); z[3] = (double)bf16hi(w.y);
    } else {
      uint32_t w = *reinterpret_cast<const uint32_t*>(src_row + 4 * lane);
      z[0] = (double)bf16lo(w); z[1] = (double)bf16hi(w);
    }
#pragma unroll
    for (int i = 0; i < P; ++i) {
      if (!isfinite(z[i])) { finite = false; z[i] = 0.0; }
    }
  } else {
#pragma unroll
    for (int i = 0; i < P; ++i) z[i] = 0.0;
  }
  finite = __all_sync(0xffffffffu, finite);

  // sum of squares, pairwise halving (uses the unrotated coordinates)
  double ss;
  if constexpr (P == 4) {
    ss = __dadd_rn(__dadd_rn(__dmul_rn(z[0], z[0]), __dmul_rn(z[1], z[1])),
                   __dadd_rn(__dmul_rn(z[2], z[2]), __dmul_rn(z[3], z[3])));
  } else {
    ss = __dadd_rn(__dmul_rn(z[0], z[0]), __dmul_rn(z[1], z[1]));
  }
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) ss = __dadd_rn(ss, __shfl_xor_sync(0xffffffffu, ss, m));

  // the tier's rotation signs: coordinate i negated before the transform (exact)
#pragma unroll
  for (int i = 0; i < P; ++i) {
    const int c = P * lane + i;
    if ((signs[c >> 5] >> (c & 31)) & 1u) z[i] = -z[i];
  }

  // in-lane butterflies (h < P)
#pragma unroll
  for (int h = 1; h < P; h <<= 1) {
#pragma unroll
    for (int j = 0; j < P; ++j) {
      if ((j & h) == 0) {
        double a = z[j], b = z[j + h];
        z[j] = __dadd_rn(a, b);
        z[j + h] = __dsub_rn(a, b);
      }
    }
  }
  // cross-lane butterflies (h >= P): partner lane l ^ (h / P)
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    const bool upper = (lane & m) != 0;
#pragma unroll
    for (int j = 0; j < P; ++j) {
      double other = __shfl_xor_sync(0xffffffffu, z[j], m);
      z[j] = upper ? __dsub_rn(other, z[j]) : __dadd_rn(z[j], other);
    }
  }

  __half s16 = __double2half(__dsqrt_rn(ss));
  double s = (double)__half2float(s16);
  const bool overflow = isinf(s);
  const bool refuse = !finite || overflow;
  if (lane == 0 && valid) {
    if (!finite) flag_error(err, AKV_EFLAG_NONFINITE);
    else if (overflow) flag_error(err, AKV_EFLAG_RANGE);
  }

  uint32_t codes = 0;
#pragma unroll
  for (int i = 0; i < P; ++i) {
    int c = 0;
#pragma unroll
    for (int j = 0; j < 15; ++j) c += (z[i] > __dmul_rn(s, bound[j])) ? 1 : 0;
    if (s == 0.0 || refuse || !valid) c = 7;
    codes |= (uint32_t)c << (4 * i);
  }
  if constexpr (P == 4) {
    *reinterpret_cast<uint16_t*>(code_row + 2 * lane) = (uint16_t)codes;
  } else {
    code_row[lane] = (uint8_t)codes;
  }
  if (lane == 0) *scale_slot = (refuse || !valid) ? (uint16_t)0 : __half_as_ushort(s16);
}

template <int D>
__global__ void __launch_bounds__(512) encode_kernel(const __grid_constant__ EncodeParams p) {
  const int item = blockIdx.x;
  const int h = blockIdx.y;
  const int bl = find_seq(p.seq, item);
  const int b = p.seq.b0 + bl;
  const int blk = item - p.seq.item_base[bl];
  const int row = threadIdx.x >> 5;
  const int tok = blk * kPageTokens + row;
  const bool valid = tok < p.seq.len[bl];
  __shared__ double bound[15];
  if (threadIdx.x < 15) bound[threadIdx.x] = p.bound[threadIdx.x];
  __syncthreads();
  const int tok0 = blk * kPageTokens;
  // destination block of K and V (all rows of the block share it)
  uint8_t* kblock = const_cast<uint8_t*>(codes_block<D>(p.dst, p.dst.k, b, h, tok0, p.err));
  uint8_t* vblock = const_cast<uint8_t*>(codes_block<D>(p.dst, p.dst.v, b, h, tok0, p.err));
  const uint8_t* ksrc = valid ? bf16_row(p.src, p.src.k, b, h, tok, p.err) : nullptr;
  const uint8_t* vsrc = valid ? bf16_row(p.src, p.src.v, b, h, tok, p.err) : nullptr;
  constexpr int ROWB = D / 2;
  // keys: the block's own row layout; values: code rows staged here, then stored by token
  // pairs (byte k of pair row r = code k of token 2r | code k of token 2r + 1 << 4) with
  // unit u of d/8 bytes at position u ^ w(r) -- the order the tensor-core product reads
  __shared__ __align__(16) uint8_t vrows[16 * ROWB];
  encode_vector<D>(ksrc, kblock + row * ROWB, reinterpret_cast<uint16_t*>(kblock + 16 * ROWB) + row, valid, bound,
                   p.dst.signs, p.err);
  encode_vector<D>(vsrc, vrows + row * ROWB, reinterpret_cast<uint16_t*>(vblock + 16 * ROWB) + row, valid, bound,
                   p.dst.signs, p.err);
  __syncthreads();
  // 8 pair rows of D bytes = 16 ROWB bytes; thread i writes 4 bytes of pair row i / (D/4)
  constexpr int US = D / 8;
  for (int i = threadIdx.x; i < 16 * ROWB / 4; i += blockDim.x) {
    const int r = i / (D / 4), k0 = 4 * (i % (D / 4));  // dims k0 .. k0 + 3 of pair row r
    const uint8_t* lo = vrows + (2 * r) * ROWB + k0 / 2;
    const uint8_t* hi = vrows + (2 * r + 1) * ROWB + k0 / 2;
    const uint32_t a = (uint32_t)lo[0] | ((uint32_t)lo[1] << 8);  // codes of dims k0..k0+3, token 2r
    const uint32_t c = (uint32_t)hi[0] | ((uint32_t)hi[1] << 8);  // token 2r + 1
    uint32_t out = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) out |= (((a >> (4 * j)) & 15u) | (((c >> (4 * j)) & 15u) << 4)) << (8 * j);
    const int w = D == 128 ? 2 * (r & 3) : 4 * ((r >> 1) & 1);
    const int u = k0 / US;
    *reinterpret_cast<uint32_t*>(vblock + r * D + (u ^ w) * US + k0 % US) = out;
  }
}

}  // namespace

cudaError_t launch_encode(const EncodeParams& p, int d, int n_items, cudaStream_t s) {
  dim3 grid(n_items, p.Hkv);
  if (d == 128) encode_kernel<128><<<grid, 512, 0, s>>>(p);
  else encode_kernel<64><<<grid, 512, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace akv

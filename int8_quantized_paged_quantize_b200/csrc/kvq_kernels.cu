// CUDA kernels of libkvq for sm_100a: quantize-on-append, the launch of the
// paged GQA decode attention kernel (kvq_decode_mma.cuh, split-K partials) and
// the log-sum-exp merge.
//
// Sources (web pages, by title and section):
//  "KV cache quantization: what FP8/INT8 K and V really give, and their limits"
//     - "What KV cache quantization actually is": quantize only when storing,
//       scale from the full BF16 values, BF16 per-token scales, dequantization
//       fused into the attention kernel right before the matmuls.
//     - "Formats you will actually meet": E4M3 for K/V; INT8 per-token
//       asymmetric (scale, zero_point).
//  "Fitting 76x concurrent requests with an FP8 KV cache" - "4. Precision
//     loss?": 8-bit storage, FP32 accumulation of the attention dot products.
//  "KV Cache compression" - "5.1 Quantization pipeline" (a separate dequant
//     kernel gives the bandwidth gain back), "6.3" (quantize right after K/V
//     are computed).
//  "From FP8 KV cache to INT4 weight-only" - "Core concepts" 1) decode reads the
//     whole cache once per step and is memory bound; 2) PagedAttention.
//
// Numerics that must match the oracle bit for bit (codes and scales):
//  IEEE f32 division (__fdiv_rn), BF16 round-to-nearest-even of the scale,
//  hardware E4M3 conversion with round-to-nearest-even and saturation, rint
//  (ties to even) for INT8. This file is compiled without fast-math.

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "kvq_internal.h"

namespace kvq {

// Per-device error word (KVQ_DEVERR_* bits), read by kvq_device_error().
__device__ unsigned int g_error_word;

__device__ __forceinline__ void flag_error(unsigned int bit) { atomicOr(&g_error_word, bit); }

// ------------------------------------------------------------------ helpers
// Byte offset, inside a K page whose token rows are ROWB bytes, of 16-byte
// chunk c of token t: tokens come in two groups of 8, and a group stores its
// chunk 0 for tokens 0..7, then chunk 1, ... (8 x 16-byte core matrices, the
// K-major operand layout of the tensor cores).
template <int ROWB>
__host__ __device__ __forceinline__ int k_chunk_offset(int c, int t) {
  return (t >> 3) * (8 * ROWB) + c * 128 + (t & 7) * 16;
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

}  // namespace kvq

#include <algorithm>
#include <utility>

#include "kvq_decode_mma.cuh"
#include "kvq_decode_kivi.cuh"
#include "kvq_kivi.cuh"
#include "kvq_merge.cuh"
#include "kvq_prefill.cuh"

namespace kvq {

// ------------------------------------------------------------------ append
// A (token, KV head) row of D BF16 values is quantized by a group of
// kRowLanes = 8 lanes with E = D/8 consecutive values each (two 16-byte loads
// at D = 128), so a warp instruction serves four rows and the per-row work
// (range, scale, reciprocal, zero point) is shared by 16 values per lane. The
// range is an integer max over the group, the BF16 scale (+ zero point) is
// formed on each of its lanes, and the lane's codes are packed little-endian
// in d order into `w`.
constexpr int kRowLanes = 8;

template <int D, int FMT>
struct RowCodes {
  static constexpr int E = D / kRowLanes;
  static constexpr int ELT = (FMT == KVQ_BF16) ? 2 : 1;
  static constexpr int WORDS = E * ELT / 4;
  uint32_t w[WORDS];
  __nv_bfloat16 s;
  int zp;
};

// This lane's D/8 BF16 values of a row, as packed pairs.
template <int D>
__device__ __forceinline__ void load_row(const __nv_bfloat16* src, uint32_t (&raw)[D / (2 * kRowLanes)]) {
#pragma unroll
  for (int c = 0; c < D / (8 * kRowLanes); ++c) {
    const uint4 u = reinterpret_cast<const uint4*>(src)[c];
    raw[4 * c] = u.x; raw[4 * c + 1] = u.y; raw[4 * c + 2] = u.z; raw[4 * c + 3] = u.w;
  }
}

// a / c for a constant c > 0 and a >= 0: RN(a * RN(1/c)) corrected once on the
// exact FMA residual. For c = 448 and c = 57344 over every BF16 a, and for
// c = 255 over every a = RN(hi - lo) of BF16 hi >= 0 >= lo, this is the IEEE
// quotient bit for bit (tests/test_scale_division.py enumerates all of them),
// so the row scales are those of a plain division.
template <int C>
__device__ __forceinline__ float div_by_const(float a) {
  constexpr float c = float(C), r = 1.0f / float(C);
  const float q = __fmul_rn(a, r);
  return __fmaf_rn(__fmaf_rn(-q, c, a), r, q);
}

// x / s for the row's BF16 scale s > 0, as the codes need it. For s >= 2^-100
// it is RN(x * RN(1/s)) corrected once on the exact FMA residual (Markstein's
// method), with the residual's sign folded so that a zero x keeps its sign
// (-0 / s = -0) without a test: it may differ from the IEEE quotient in the
// last bit, but the E4M3, E5M2 and rint codes taken from it are the IEEE
// quotient's for every BF16 x with |x| <= 65536 s, subnormal x included
// (enumerated by tests/test_scale_division.py). Rows with a smaller scale take
// the IEEE division.
struct ScaleDiv {
  float s, r;
  bool fast;
  __device__ __forceinline__ explicit ScaleDiv(float s_) {
    s = s_;
    fast = s_ >= 7.88860905e-31f;                   // 2^-100
    r = fast ? __frcp_rn(s_) : 0.f;
  }
  __device__ __forceinline__ float operator()(float x) const {
    if (!fast) return __fdiv_rn(x, s);
    const float q = __fmul_rn(x, r);
    const float e = __fmaf_rn(q, s, -x);             // minus the residual x - q s (exact)
    return __fmaf_rn(-e, r, q);
  }
};

// Integer rounding by one addition: for |q| < 2^22, q + 1.5 * 2^23 lies in
// [2^23, 2^24), where the float spacing is 1, so the sum is rint(q) (round to
// nearest even) and its bit pattern is kRintBits + rint(q).
constexpr float kRintMagic = 12582912.0f;
constexpr int kRintBits = 0x4B400000;

// The low bytes of four ints, packed little-endian.
__device__ __forceinline__ uint32_t pack_low_bytes(int a, int b, int c, int d) {
  const uint32_t lo = __byte_perm(uint32_t(a), uint32_t(b), 0x0040);
  const uint32_t hi = __byte_perm(uint32_t(c), uint32_t(d), 0x0040);
  return __byte_perm(lo, hi, 0x5410);
}


// Lane-wise max of two pairs of 16-bit fields, unsigned or signed (the
// signed form with a floor of 0).
__device__ __forceinline__ uint32_t vmax_u16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t vmax_relu_s16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.relu.s16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Field-wise max of a u16x2 word over the kRowLanes lanes of this row group
// (the four groups of the warp reduce at once).
__device__ __forceinline__ uint32_t row_vmax_u16x2(uint32_t v) {
#pragma unroll
  for (int o = kRowLanes / 2; o > 0; o >>= 1) v = vmax_u16x2(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// The two BF16 values of a packed pair as floats (low half first).
__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t w) { return make_float2(bf16_lo(w), bf16_hi(w)); }

// Markstein's corrected quotient on a pair: q = RN(x r), e = RN(q s - x)
// (exact), q' = RN(q - e r), with -x and -r passed in so that a zero x keeps
// its sign; the same arithmetic as ScaleDiv, two lanes per instruction.
__device__ __forceinline__ float2 div_pair(float2 x, float2 r2, float2 nr2, float2 s2) {
  const float2 nx = __fmul2_rn(x, make_float2(-1.f, -1.f));
  const float2 q = __fmul2_rn(x, r2);
  const float2 e = __ffma2_rn(q, s2, nx);
  return __ffma2_rn(e, nr2, q);
}

// Two pairs of quotients as four E4M3 / E5M2 codes (RNE, satfinite),
// little-endian: a.x in the low byte.
template <bool E4>
__device__ __forceinline__ uint32_t fp8x4(float2 a, float2 b) {
  uint32_t w;
  if constexpr (E4)
    asm("{\n .reg .b16 lo, hi;\n cvt.rn.satfinite.e4m3x2.f32 lo, %2, %1;\n"
        " cvt.rn.satfinite.e4m3x2.f32 hi, %4, %3;\n mov.b32 %0, {lo, hi};\n}"
        : "=r"(w) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  else
    asm("{\n .reg .b16 lo, hi;\n cvt.rn.satfinite.e5m2x2.f32 lo, %2, %1;\n"
        " cvt.rn.satfinite.e5m2x2.f32 hi, %4, %3;\n mov.b32 %0, {lo, hi};\n}"
        : "=r"(w) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return w;
}

// Two ints saturated to [-128, 127] in bytes 0 (b) and 1 (a), bytes 2-3 from
// the low half of c.
__device__ __forceinline__ uint32_t pack_sat_s8x2(int a, int b, uint32_t c) {
  uint32_t d;
  asm("cvt.pack.sat.s8.s32.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// The row maximum is taken on bit patterns: non-negative floats (and BF16
// values) order as their bits read as integers and every negative one (-0
// included) reads as a negative signed integer, so an integer max with a floor
// of 0 gives the float maximum, +0 when nothing is positive. The lane's BF16
// pairs are reduced as 16-bit fields, two values per instruction. Every lane
// of the warp must call the quantizers (the half-warp reductions are warp-wide
// shuffles); a row that is not stored is still quantized, from whatever its
// lanes hold.
template <int D, int FMT>
__device__ __forceinline__ void quantize_row(const uint32_t (&raw)[D / (2 * kRowLanes)], RowCodes<D, FMT>& rc) {
  constexpr int E = D / kRowLanes;
  constexpr int NW = E / 2;                          // BF16 pairs of the lane
  rc.zp = 0;
  rc.s = __float2bfloat16_rn(0.f);
  if constexpr (FMT == KVQ_BF16) {
#pragma unroll
    for (int i = 0; i < NW; ++i) rc.w[i] = raw[i];
    return;
  } else {
#pragma unroll
    for (int i = 0; i < RowCodes<D, FMT>::WORDS; ++i) rc.w[i] = 0u;
    if constexpr (FMT == KVQ_FP8_E4M3 || FMT == KVQ_FP8_E5M2) {
      // s = bf16(amax / max code), code = fp8_rne_satfinite(x / s)
      constexpr bool E4 = FMT == KVQ_FP8_E4M3;
      uint32_t m = raw[0] & 0x7fff7fffu;             // |x| of both halves
#pragma unroll
      for (int i = 1; i < NW; ++i) m = vmax_u16x2(m, raw[i] & 0x7fff7fffu);
      m = row_vmax_u16x2(m);
      const float amax = __uint_as_float(max(m & 0xffffu, m >> 16) << 16);
      rc.s = __float2bfloat16_rn(E4 ? div_by_const<448>(amax) : div_by_const<57344>(amax));
      const float s = __bfloat162float(rc.s);
      if (s >= 7.88860905e-31f) {                    // 2^-100: the corrected quotient
        const float r = __frcp_rn(s);
        const float2 r2 = make_float2(r, r), nr2 = make_float2(-r, -r), s2 = make_float2(s, s);
#pragma unroll
        for (int i = 0; i < NW; i += 2)
          rc.w[i >> 1] = fp8x4<E4>(div_pair(bf16x2_to_float2(raw[i]), r2, nr2, s2),
                                   div_pair(bf16x2_to_float2(raw[i + 1]), r2, nr2, s2));
      } else if (s != 0.f) {                         // tiny scale: the IEEE quotient
#pragma unroll
        for (int i = 0; i < NW; i += 2) {
          const float2 a = bf16x2_to_float2(raw[i]), b = bf16x2_to_float2(raw[i + 1]);
          rc.w[i >> 1] = fp8x4<E4>(make_float2(__fdiv_rn(a.x, s), __fdiv_rn(a.y, s)),
                                   make_float2(__fdiv_rn(b.x, s), __fdiv_rn(b.y, s)));
        }
      }
    } else {  // INT8 asymmetric: range [lo, hi] widened to hold 0
      // hi = max(0, max x) and nlo = max(0, max -x), as 16-bit fields
      uint32_t hw = vmax_relu_s16x2(raw[0], 0u), nw = vmax_relu_s16x2(raw[0] ^ 0x80008000u, 0u);
#pragma unroll
      for (int i = 1; i < NW; ++i) {
        hw = vmax_relu_s16x2(hw, raw[i]);
        nw = vmax_relu_s16x2(nw, raw[i] ^ 0x80008000u);
      }
      // both maxima in one word (hi low, nlo high), reduced over the row group
      const uint32_t hn = row_vmax_u16x2(vmax_u16x2(__byte_perm(hw, nw, 0x5410),
                                                     __byte_perm(hw, nw, 0x7632)));
      const float hi = bf16_lo(hn), nlo = bf16_hi(hn);
      rc.s = __float2bfloat16_rn(div_by_const<255>(__fadd_rn(hi, nlo)));
      const float s = __bfloat162float(rc.s);
      if (s != 0.f) {
        const ScaleDiv div(s);
        const float zq = fminf(fmaxf(-div(nlo), -1024.f), 1024.f);   // lo / s
        rc.zp = min(127, max(-128, -128 - __float2int_rn(zq)));
        // code = clamp(rint(x / s) + zp, -128, 127): every x of the row lies in
        // [lo, hi], so |x / s| stays near 255 and the rounding addition
        // applies; the sum's bits less kRintBits are rint(x / s), zp is added
        // as an integer and the pack saturates
        const int off = rc.zp - kRintBits;
        int c[E];
        if (div.fast) {
          const float2 r2 = make_float2(div.r, div.r), nr2 = make_float2(-div.r, -div.r);
          const float2 s2 = make_float2(s, s), mg = make_float2(kRintMagic, kRintMagic);
#pragma unroll
          for (int i = 0; i < NW; ++i) {
            const float2 t = __fadd2_rn(div_pair(bf16x2_to_float2(raw[i]), r2, nr2, s2), mg);
            c[2 * i] = __float_as_int(t.x) + off;
            c[2 * i + 1] = __float_as_int(t.y) + off;
          }
        } else {
#pragma unroll
          for (int i = 0; i < NW; ++i) {
            const float2 x = bf16x2_to_float2(raw[i]);
            c[2 * i] = __float_as_int(__fadd_rn(__fdiv_rn(x.x, s), kRintMagic)) + off;
            c[2 * i + 1] = __float_as_int(__fadd_rn(__fdiv_rn(x.y, s), kRintMagic)) + off;
          }
        }
#pragma unroll
        for (int i = 0; i < E; i += 4) rc.w[i >> 2] = pack_sat_s8x2(c[i + 1], c[i], pack_sat_s8x2(c[i + 3], c[i + 2], 0u));
      }
    }
  }
}

// Static-scale INT8 (one given scale per channel, or one per cache): code =
// clamp(rint(x / s), -127, 127), 0 where s <= 0 or s is NaN. sc[i] and rc_[i]
// (shared memory) are the scale of this lane's element i and its reciprocal
// RN(1/s), 0 when s is below 2^-100 (those take the IEEE division). x is first clamped to
// +-65536 s, which changes only quotients that saturate anyway and keeps the
// corrected quotient inside the range where its rint equals that of the IEEE
// quotient (tests/test_scale_division.py).
template <int D>
__device__ __forceinline__ void quantize_row_static(const uint32_t (&raw)[D / (2 * kRowLanes)],
                                                    const float* sc, const float* rc_,
                                                    RowCodes<D, KVQ_INT8_CHANNEL>& rc) {
  constexpr int E = D / kRowLanes;
  rc.zp = 0;
  rc.s = __float2bfloat16_rn(0.f);
#pragma unroll
  for (int i = 0; i < RowCodes<D, KVQ_INT8_CHANNEL>::WORDS; ++i) rc.w[i] = 0u;
  // the lane's scales and reciprocals as 16-byte reads (sc, rc_ are 64-byte aligned)
  float scv[E], rcv[E];
#pragma unroll
  for (int i = 0; i < E; i += 4) {
    const float4 a = *reinterpret_cast<const float4*>(sc + i);
    const float4 b = *reinterpret_cast<const float4*>(rc_ + i);
    scv[i] = a.x; scv[i + 1] = a.y; scv[i + 2] = a.z; scv[i + 3] = a.w;
    rcv[i] = b.x; rcv[i + 1] = b.y; rcv[i + 2] = b.z; rcv[i + 3] = b.w;
  }
  int c[E];
#pragma unroll
  for (int i = 0; i < E; ++i) {
    const float x = (i & 1) ? bf16_hi(raw[i / 2]) : bf16_lo(raw[i / 2]);
    const float s = scv[i], r = rcv[i];
    c[i] = 0;
    if (s > 0.f) {
      const float lim = s * 65536.f;
      const float xc = fminf(fmaxf(x, -lim), lim);
      float q;
      if (r != 0.f) {
        const float q0 = __fmul_rn(xc, r);
        const float e = __fmaf_rn(q0, s, -xc);
        q = __fmaf_rn(-e, r, q0);
      } else {
        q = __fdiv_rn(xc, s);
      }
      // |q| <= 65536 (x clamped above): the rounding addition applies
      c[i] = min(kRintBits + 127, max(kRintBits - 127, __float_as_int(__fadd_rn(q, kRintMagic))));
    }
  }
#pragma unroll
  for (int i = 0; i < E; i += 4) rc.w[i >> 2] = pack_low_bytes(c[i], c[i + 1], c[i + 2], c[i + 3]);
}

// Bytes [p, e) of the 16-byte chunk at dst (16-byte aligned) from w, with the
// widest aligned stores the range allows: one 16-byte store for a whole chunk,
// else 8-, 4-, 2- and 1-byte pieces. Bytes outside [p, e) are not touched, so
// writers of disjoint byte ranges of one chunk never clobber each other.
__device__ __forceinline__ void store_bytes16(uint8_t* dst, const uint32_t (&w)[4], int p, int e) {
  if (p == 0 && e == 16) {
    *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
    return;
  }
#pragma unroll
  for (int h8 = 0; h8 < 2; ++h8) {
    const int a8 = max(p, 8 * h8), b8 = min(e, 8 * h8 + 8);
    if (a8 >= b8) continue;
    if (a8 == 8 * h8 && b8 == 8 * h8 + 8) {
      *reinterpret_cast<uint2*>(dst + 8 * h8) = make_uint2(w[2 * h8], w[2 * h8 + 1]);
      continue;
    }
#pragma unroll
    for (int h4 = 0; h4 < 2; ++h4) {
      const int base4 = 8 * h8 + 4 * h4;
      const int a4 = max(a8, base4), b4 = min(b8, base4 + 4);
      if (a4 >= b4) continue;
      const uint32_t word = w[2 * h8 + h4];
      if (a4 == base4 && b4 == base4 + 4) {
        *reinterpret_cast<uint32_t*>(dst + base4) = word;
        continue;
      }
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        const int base2 = base4 + 2 * h2;
        const int a2 = max(a4, base2), b2 = min(b4, base2 + 2);
        if (a2 >= b2) continue;
        const uint32_t half = word >> (16 * h2);
        if (a2 == base2 && b2 == base2 + 2)
          *reinterpret_cast<uint16_t*>(dst + base2) = uint16_t(half);
        else
          dst[a2] = uint8_t(half >> (8 * (a2 - base2)));
      }
    }
  }
}

// One CTA of 8 warps per (16 consecutive input tokens, KV head). Warp w takes
// tokens 2w and 2w+1: its four lane groups quantize their K rows (lanes 0-15)
// and V rows (lanes 16-31) into shared memory in one pass. The input rows are
// requested before the slots arrive (a skipped token's row is read and
// dropped), so the loads overlap. The window is then written in page-sized
// pieces:
//   - the 16 tokens fill one page in order (the bulk / prefill case): the page
//     is written as whole 16-byte chunks, K in its chunk-major layout and V
//     transposed with byte permutes;
//   - otherwise each token writes its K chunks, and the tokens are grouped into
//     segments (runs of consecutive slots inside one page); a segment writes its
//     byte range of each transposed V chunk once, with the widest aligned
//     stores that range allows. A page continued from an offset (chunked
//     prefill) thus costs one partial chunk per channel, not one byte store per
//     token and channel.
// Register use is capped at 32 so that 8 CTAs (64 warps) fit on an SM (a few
// bytes of spills for INT8 with its zero point cost less than 6 CTAs did); the
// static-scale format takes 48 (5 CTAs), its scales in shared memory.
template <int D, int FMT>
__global__ void __launch_bounds__(256, FMT == KVQ_INT8_CHANNEL ? 5 : 8)
append_kernel(const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
              const int64_t* __restrict__ slots, int T, int Hk, int NB, uint8_t* __restrict__ kc,
              uint8_t* __restrict__ vc, __nv_bfloat16* __restrict__ ks, __nv_bfloat16* __restrict__ vs,
              int per_tensor) {
  using RC = RowCodes<D, FMT>;
  constexpr int E = RC::E, ELT = RC::ELT;
  constexpr int ROWB = D * ELT;                 // bytes of one token row
  constexpr int PADB = ROWB + 16;               // padded smem row (bank spread)
  constexpr int PAGEB = kBlockSize * ROWB;
  constexpr int NC = ROWB / 16;                 // 16-byte chunks of a K row
  constexpr int UC = ELT;                       // 16-byte V chunks per channel
  constexpr int TPC = 16 / ELT;                 // tokens per V chunk
  constexpr int MV = (FMT == KVQ_FP8_E4M3 || FMT == KVQ_FP8_E5M2) ? 1 : (FMT == KVQ_INT8_ASYM ? 2 : 0);
  __shared__ __align__(16) uint8_t kbuf[kBlockSize * PADB];
  __shared__ __align__(16) uint8_t vbuf[kBlockSize * PADB];
  __shared__ __nv_bfloat16 kmb[kBlockSize][2], vmb[kBlockSize][2];
  __shared__ int64_t sl[kBlockSize];
  __shared__ int seg_i0[kBlockSize], seg_len[kBlockSize], nseg, page_fast;
  // static scales of the head's K (0) and V (1) channels and their reciprocals
  __shared__ __align__(16) float sscale[FMT == KVQ_INT8_CHANNEL ? 2 * D : 4];
  __shared__ __align__(16) float srcp[FMT == KVQ_INT8_CHANNEL ? 2 * D : 4];

  // the decode kernel of the step may start its set-up now; it reads the
  // cache only after this grid has finished
  tc::grid_dep_launch_dependents();
  const int h = blockIdx.y;
  const int64_t tb = int64_t(blockIdx.x) * kBlockSize;
  const int n = int(min(int64_t(kBlockSize), int64_t(T) - tb));
  const int64_t nslots = int64_t(NB) * kBlockSize;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // lane group g = lane / 8: the K row (g = 0, 1) or the V row (g = 2, 3) of
  // token 2 warp + (g & 1); requested before the slots arrive
  const int which = lane >> 4;                  // 0: K row, 1: V row
  const int ti = 2 * warp + ((lane >> 3) & 1);  // token of the window
  const int d0 = (lane & (kRowLanes - 1)) * E;
  const __nv_bfloat16* src = (which ? v : k) + ((tb + ti) * Hk + h) * D + d0;
  uint32_t raw[D / (2 * kRowLanes)];
#pragma unroll
  for (int e = 0; e < D / (2 * kRowLanes); ++e) raw[e] = 0u;
  if (ti < n) load_row<D>(src, raw);
  if (threadIdx.x < kBlockSize) sl[threadIdx.x] = threadIdx.x < n ? slots[tb + threadIdx.x] : -1;
  if constexpr (FMT == KVQ_INT8_CHANNEL) {
    for (int i = threadIdx.x; i < 2 * D; i += blockDim.x) {
      const float sv = __bfloat162float((i >= D ? vs : ks)[per_tensor ? 0 : h * D + i % D]);
      sscale[i] = sv;
      srcp[i] = sv >= 7.88860905e-31f ? __frcp_rn(sv) : 0.f;   // 2^-100
    }
  }
  __syncthreads();

  if (warp == 0) {
    const int64_t si = lane < kBlockSize ? sl[lane] : -1;
    const int64_t sp = (lane > 0 && lane < kBlockSize) ? sl[lane - 1] : -1;
    const int64_t s0 = sl[0];
    // whole page in order: slot i = s0 + i for all 16 tokens, s0 page-aligned
    const bool inpage = lane >= kBlockSize || (si == s0 + lane && s0 >= 0 && s0 % kBlockSize == 0 &&
                                               s0 < nslots && n == kBlockSize);
    const bool fast = __all_sync(0xffffffffu, inpage);
    // segments: a token starts one unless it continues the previous token's
    // slot inside the same page
    const bool valid = si >= 0 && si < nslots;
    const bool start = valid && !(sp >= 0 && sp < nslots && si == sp + 1 && si % kBlockSize != 0);
    const unsigned vmask = __ballot_sync(0xffffffffu, valid);
    const unsigned smask = __ballot_sync(0xffffffffu, start);
    if (start) {
      const int idx = __popc(smask & ((1u << lane) - 1u));
      // the run ends at the next start or at the first invalid token
      const unsigned stop = (smask | ~vmask) & ~((2u << lane) - 1u);
      seg_i0[idx] = lane;
      seg_len[idx] = (stop ? __ffs(stop) - 1 : 32) - lane;
    }
    if (lane == 0) {
      nseg = __popc(smask);
      page_fast = fast;
    }
  }

  {
    // every lane quantizes (the reductions span the warp); only real rows store
    RC rc;
    if constexpr (FMT == KVQ_INT8_CHANNEL)
      quantize_row_static<D>(raw, sscale + which * D + d0, srcp + which * D + d0, rc);
    else quantize_row<D, FMT>(raw, rc);
    const int64_t slot = ti < n ? sl[ti] : -1;
    if (slot >= nslots) {
      if ((lane & (kRowLanes - 1)) == 0) flag_error(KVQ_DEVERR_SLOT);
    } else if (slot >= 0) {
      uint8_t* dst = (which ? vbuf : kbuf) + ti * PADB + d0 * ELT;
#pragma unroll
      for (int c = 0; c < E * ELT / 16; ++c)
        reinterpret_cast<uint4*>(dst)[c] = make_uint4(rc.w[4 * c], rc.w[4 * c + 1], rc.w[4 * c + 2], rc.w[4 * c + 3]);
      if constexpr (E * ELT == 8) *reinterpret_cast<uint2*>(dst) = make_uint2(rc.w[0], rc.w[1]);
      if ((lane & (kRowLanes - 1)) == 0) {
        (which ? vmb : kmb)[ti][0] = rc.s;
        (which ? vmb : kmb)[ti][1] = __int2bfloat16_rn(rc.zp);
      }
    }
  }
  __syncthreads();

  if (page_fast) {                                   // uniform over the CTA
    const int64_t page = (sl[0] / kBlockSize) * Hk + h;
    uint8_t* kp = kc + page * PAGEB;
    uint8_t* vp = vc + page * PAGEB;
    // items [0, KN): K chunk j = (token group t/8, c, t%8) <- bytes [16c, 16c+16)
    // of token t's row. Items [KN, KN + VN): a V piece, from 32-bit words of
    // the staged rows transposed with byte permutes.
    constexpr int KN = PAGEB / 16;
    constexpr int VN = ELT == 1 ? 2 * (D / 4) : 2 * (D / 2);
    for (int j = threadIdx.x; j < KN + VN; j += blockDim.x) {
      if (j < KN) {
        const int c = (j >> 3) % NC, t = (j / (8 * NC)) * 8 + (j & 7);
        *reinterpret_cast<uint4*>(kp + j * 16) = *reinterpret_cast<const uint4*>(kbuf + t * PADB + c * 16);
        continue;
      }
      const int jv = j - KN;
      if constexpr (ELT == 1) {
        // channels 4c..4c+3, tokens 8h..8h+7: two 4x4 byte transposes; the
        // result is the low or high 8 bytes of four channels' chunks
        const int c = jv % (D / 4), hh = jv / (D / 4);
        uint32_t o[4][2];
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          const int t0 = 8 * hh + 4 * g;
          const uint32_t r0 = *reinterpret_cast<const uint32_t*>(vbuf + (t0 + 0) * PADB + 4 * c);
          const uint32_t r1 = *reinterpret_cast<const uint32_t*>(vbuf + (t0 + 1) * PADB + 4 * c);
          const uint32_t r2 = *reinterpret_cast<const uint32_t*>(vbuf + (t0 + 2) * PADB + 4 * c);
          const uint32_t r3 = *reinterpret_cast<const uint32_t*>(vbuf + (t0 + 3) * PADB + 4 * c);
          const uint32_t a01 = __byte_perm(r0, r1, 0x5140), a23 = __byte_perm(r2, r3, 0x5140);
          const uint32_t b01 = __byte_perm(r0, r1, 0x7362), b23 = __byte_perm(r2, r3, 0x7362);
          o[0][g] = __byte_perm(a01, a23, 0x5410);
          o[1][g] = __byte_perm(a01, a23, 0x7632);
          o[2][g] = __byte_perm(b01, b23, 0x5410);
          o[3][g] = __byte_perm(b01, b23, 0x7632);
        }
#pragma unroll
        for (int m = 0; m < 4; ++m)
          *reinterpret_cast<uint2*>(vp + (4 * c + m) * 16 + 8 * hh) = make_uint2(o[m][0], o[m][1]);
      } else {
        // channels 2c, 2c+1, tokens 8u..8u+7: 2x2 transposes of 16-bit halves
        const int c = jv % (D / 2), u = jv / (D / 2);
        uint32_t lo4[4], hi4[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int t0 = 8 * u + 2 * q;
          const uint32_t w0 = *reinterpret_cast<const uint32_t*>(vbuf + t0 * PADB + 4 * c);
          const uint32_t w1 = *reinterpret_cast<const uint32_t*>(vbuf + (t0 + 1) * PADB + 4 * c);
          lo4[q] = __byte_perm(w0, w1, 0x5410);
          hi4[q] = __byte_perm(w0, w1, 0x7632);
        }
        *reinterpret_cast<uint4*>(vp + (u * D + 2 * c) * 16) = make_uint4(lo4[0], lo4[1], lo4[2], lo4[3]);
        *reinterpret_cast<uint4*>(vp + (u * D + 2 * c + 1) * 16) = make_uint4(hi4[0], hi4[1], hi4[2], hi4[3]);
      }
    }
  } else {
    // K: whole 16-byte chunks of each token's row
    for (int j = threadIdx.x; j < n * NC; j += blockDim.x) {
      const int i = j / NC, c = j % NC;
      const int64_t slot = sl[i];
      if (slot < 0 || slot >= nslots) continue;
      const int64_t page = (slot / kBlockSize) * Hk + h;
      *reinterpret_cast<uint4*>(kc + page * PAGEB + k_chunk_offset<ROWB>(c, int(slot % kBlockSize))) =
          *reinterpret_cast<const uint4*>(kbuf + i * PADB + c * 16);
    }
    // V: per (segment, channel d, chunk u) the segment's bytes of that chunk
    const int ns = nseg;
    for (int j = threadIdx.x; j < ns * D * UC; j += blockDim.x) {
      const int sg = j / (D * UC), d = (j / UC) % D, u = j % UC;
      const int i0 = seg_i0[sg], len = seg_len[sg];
      const int64_t slot0 = sl[i0];
      const int o0 = int(slot0 % kBlockSize);
      // token offsets of the segment inside chunk u
      const int ta = max(o0, u * TPC), tz = min(o0 + len, (u + 1) * TPC);
      if (ta >= tz) continue;
      uint8_t* chunk = vc + ((slot0 / kBlockSize) * Hk + h) * PAGEB + (u * D + d) * 16;
      if (tz - ta == 1) {                            // one token: one element
        const int i = i0 + (ta - o0), b = (ta - u * TPC) * ELT;
        if constexpr (ELT == 1) chunk[b] = vbuf[i * PADB + d];
        else *reinterpret_cast<uint16_t*>(chunk + b) = *reinterpret_cast<const uint16_t*>(vbuf + i * PADB + 2 * d);
        continue;
      }
      uint32_t wv[4];
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        uint32_t word = 0;
        const int w0 = u * TPC + q4 * (4 / ELT);      // first token offset of this word
        if (w0 + 4 / ELT > ta && w0 < tz) {
#pragma unroll
          for (int bb = 0; bb < 4 / ELT; ++bb) {
            const int t = w0 + bb;
            if (t >= ta && t < tz) {
              const int i = i0 + (t - o0);
              if constexpr (ELT == 1)
                word |= uint32_t(vbuf[i * PADB + d]) << (8 * bb);
              else
                word |= uint32_t(*reinterpret_cast<const uint16_t*>(vbuf + i * PADB + 2 * d)) << (16 * bb);
            }
          }
        }
        wv[q4] = word;
      }
      store_bytes16(chunk, wv, (ta - u * TPC) * ELT, (tz - u * TPC) * ELT);
    }
  }
  // metadata: one thread per (token, K or V)
  if (MV > 0 && threadIdx.x < 2 * kBlockSize) {
    const int t = threadIdx.x & 15;
    const int64_t slot = sl[t];
    if (t < n && slot >= 0 && slot < nslots) {
      const bool isv = threadIdx.x >= kBlockSize;
      __nv_bfloat16* meta = isv ? vs : ks;
      const __nv_bfloat16 (*mb)[2] = isv ? vmb : kmb;
      const int64_t row = ((slot / kBlockSize) * Hk + h) * kBlockSize + slot % kBlockSize;
      if (MV == 1) {
        meta[row] = mb[t][0];
      } else {
        *reinterpret_cast<__nv_bfloat162*>(meta + row * 2) = __halves2bfloat162(mb[t][0], mb[t][1]);
      }
    }
  }
}

// ------------------------------------------------------------------ launchers
namespace {
constexpr float kLog2e = 1.4426950408889634f;

// Launch as the programmatic dependent of the kernel ahead on the stream: it
// may start (and run up to its grid_dep_wait) before that kernel finishes.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

template <int D, int FMT>
cudaError_t append_dispatch(const void* k, const void* v, const int64_t* slots, int32_t T, void* kc,
                            void* vc, void* ks, void* vs, const kvq_dims& d, int per_tensor,
                            cudaStream_t st) {
  const dim3 grid(unsigned((int64_t(T) + kBlockSize - 1) / kBlockSize), unsigned(d.n_kv_heads));
  append_kernel<D, FMT><<<grid, 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v), slots, T,
      d.n_kv_heads, d.num_blocks, static_cast<uint8_t*>(kc), static_cast<uint8_t*>(vc),
      static_cast<__nv_bfloat16*>(ks), static_cast<__nv_bfloat16*>(vs), per_tensor);
  return cudaGetLastError();
}

template <int D, int G, int FMT>
cudaError_t decode_mma_dispatch3(const void* q, int32_t B, const void* kc, const void* vc,
                                 const void* ks, const void* vs, const int32_t* tables,
                                 const int32_t* ctx, int32_t max_ctx, float sm_scale,
                                 const DecodePlan& plan, void* ws, const kvq_dims& d,
                                 int per_tensor, int n_query, int nrg, cudaStream_t st) {
  using C = MmaCfg<D, G, FMT>;
  auto kern = decode_mma_kernel<D, G, FMT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                           int(cudaSharedmemCarveoutMaxShared));
  if (e != cudaSuccess) return e;
  // resident CTAs per SM: shared memory bounds it (registers are capped so
  // that two 8-bit CTAs fit); the BF16 ring takes a whole SM
  int dev = 0, smem_sm = 0, reserved = 0;
  e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
  if (e != cudaSuccess) return e;
  const int per_sm = std::max(1, std::min(FMT == KVQ_BF16 ? 1 : 2, smem_sm / (C::SMEM + reserved)));
  float* po = static_cast<float*>(ws);
  float* pml = reinterpret_cast<float*>(static_cast<char*>(ws) + plan.o_bytes);
  int32_t* pcnt = reinterpret_cast<int32_t*>(static_cast<char*>(ws) + plan.o_bytes + plan.ml_bytes);
  // one CTA per resident slot, in groups of nrg (one CTA per row group) that
  // walk the same share of the tile list; at least one group
  const int64_t slots_resident = int64_t(device_sm_count()) * per_sm;
  const int64_t grid = std::max<int64_t>(1, slots_resident / nrg) * nrg;
  e = launch_pdl(kern, dim3(unsigned(grid)), dim3(192), C::SMEM, st,
      static_cast<const __nv_bfloat16*>(q), static_cast<const uint8_t*>(kc),
      static_cast<const uint8_t*>(vc), static_cast<const __nv_bfloat16*>(ks),
      static_cast<const __nv_bfloat16*>(vs), tables, ctx, B, d.n_kv_heads, nrg, d.num_blocks,
      d.max_blocks_per_seq, max_ctx, plan.partition / kTileTokens, plan.slots, sm_scale * kLog2e,
      per_tensor, n_query, decode_wait_limit(), po, pml, pcnt);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int D, int FMT>
cudaError_t decode_dispatch2(int R, const void* q, int32_t B, const void* kc, const void* vc,
                             const void* ks, const void* vs, const int32_t* tables,
                             const int32_t* ctx, int32_t max_ctx, float sm_scale,
                             const DecodePlan& plan, void* ws, const kvq_dims& d, int per_tensor,
                             int n_query, cudaStream_t st) {
  // R query rows per KV head, taken in groups of gp rows (one instantiation per gp)
  int gp = 1;
  const int nrg = row_groups(R, &gp);
  switch (gp) {
    case 1: return decode_mma_dispatch3<D, 1, FMT>(q, B, kc, vc, ks, vs, tables, ctx, max_ctx, sm_scale, plan, ws, d, per_tensor, n_query, nrg, st);
    case 2: return decode_mma_dispatch3<D, 2, FMT>(q, B, kc, vc, ks, vs, tables, ctx, max_ctx, sm_scale, plan, ws, d, per_tensor, n_query, nrg, st);
    case 4: return decode_mma_dispatch3<D, 4, FMT>(q, B, kc, vc, ks, vs, tables, ctx, max_ctx, sm_scale, plan, ws, d, per_tensor, n_query, nrg, st);
    default: return decode_mma_dispatch3<D, 8, FMT>(q, B, kc, vc, ks, vs, tables, ctx, max_ctx, sm_scale, plan, ws, d, per_tensor, n_query, nrg, st);
  }
}

template <int D, int FMT>
cudaError_t prefill_dispatch2(const void* q, int32_t B, const void* kc, const void* vc,
                              const void* ks, const void* vs, const int32_t* tables,
                              const int32_t* ctx, int32_t max_ctx, float sm_scale,
                              const DecodePlan& plan, void* ws, const kvq_dims& d, int per_tensor,
                              int n_query, cudaStream_t st) {
  using C = PfCfg<D, FMT>;
  auto kern = prefill_mma_kernel<D, FMT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const int G = d.n_q_heads / d.n_kv_heads;
  const int R = G * n_query;                         // query rows of a KV head
  const int nrb = (R + 127) / 128;                   // 128-row blocks, one CTA each
  float* po = static_cast<float*>(ws);
  float* pml = reinterpret_cast<float*>(static_cast<char*>(ws) + plan.o_bytes);
  int32_t* pcnt = reinterpret_cast<int32_t*>(static_cast<char*>(ws) + plan.o_bytes + plan.ml_bytes);
  // one CTA per SM, in groups of nrb that walk the same share of the tile list
  const int64_t grid = std::max<int64_t>(1, int64_t(device_sm_count()) / nrb) * nrb;
  e = launch_pdl(kern, dim3(unsigned(grid)), dim3(448), C::SMEM, st,
      static_cast<const __nv_bfloat16*>(q), static_cast<const uint8_t*>(kc),
      static_cast<const uint8_t*>(vc), static_cast<const __nv_bfloat16*>(ks),
      static_cast<const __nv_bfloat16*>(vs), tables, ctx, B, d.n_kv_heads, G, n_query, nrb,
      d.num_blocks, d.max_blocks_per_seq, max_ctx, plan.partition / kTileTokens, plan.slots,
      sm_scale * kLog2e, per_tensor, decode_wait_limit(), po, pml, pcnt);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}
}  // namespace

int launch_prefill_partial(const void* q, int32_t B, const void* kc, const void* vc,
                           const void* ks, const void* vs, const int32_t* tables,
                           const int32_t* ctx, int32_t max_ctx, float sm_scale,
                           const DecodePlan& plan, void* ws, kvq_fmt fmt, const kvq_dims& d,
                           void* stream, int n_query) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  const int pt = fmt == KVQ_INT8_TENSOR;
#define KVQ_PF(DD, FF) prefill_dispatch2<DD, FF>(q, B, kc, vc, ks, vs, tables, ctx, max_ctx, sm_scale, plan, ws, d, pt, n_query, st)
  if (d.head_dim == 128) {
    if (fmt == KVQ_FP8_E4M3) e = KVQ_PF(128, KVQ_FP8_E4M3);
    else if (fmt == KVQ_FP8_E5M2) e = KVQ_PF(128, KVQ_FP8_E5M2);
    else if (fmt == KVQ_INT8_ASYM) e = KVQ_PF(128, KVQ_INT8_ASYM);
    else if (fmt_static(fmt)) e = KVQ_PF(128, KVQ_INT8_CHANNEL);
    else e = KVQ_PF(128, KVQ_BF16);
  } else {
    if (fmt == KVQ_FP8_E4M3) e = KVQ_PF(64, KVQ_FP8_E4M3);
    else if (fmt == KVQ_FP8_E5M2) e = KVQ_PF(64, KVQ_FP8_E5M2);
    else if (fmt == KVQ_INT8_ASYM) e = KVQ_PF(64, KVQ_INT8_ASYM);
    else if (fmt_static(fmt)) e = KVQ_PF(64, KVQ_INT8_CHANNEL);
    else e = KVQ_PF(64, KVQ_BF16);
  }
#undef KVQ_PF
  return int(e);
}

int launch_append(const void* k, const void* v, const int64_t* slots, int32_t T, void* kc,
                  void* vc, void* ks, void* vs, kvq_fmt fmt, const kvq_dims& d, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int pt = fmt == KVQ_INT8_TENSOR;
  cudaError_t e;
#define KVQ_APP(DD, FF) append_dispatch<DD, FF>(k, v, slots, T, kc, vc, ks, vs, d, pt, st)
  if (d.head_dim == 128) {
    if (fmt == KVQ_FP8_E4M3) e = KVQ_APP(128, KVQ_FP8_E4M3);
    else if (fmt == KVQ_FP8_E5M2) e = KVQ_APP(128, KVQ_FP8_E5M2);
    else if (fmt == KVQ_INT8_ASYM) e = KVQ_APP(128, KVQ_INT8_ASYM);
    else if (fmt_static(fmt)) e = KVQ_APP(128, KVQ_INT8_CHANNEL);
    else e = KVQ_APP(128, KVQ_BF16);
  } else {
    if (fmt == KVQ_FP8_E4M3) e = KVQ_APP(64, KVQ_FP8_E4M3);
    else if (fmt == KVQ_FP8_E5M2) e = KVQ_APP(64, KVQ_FP8_E5M2);
    else if (fmt == KVQ_INT8_ASYM) e = KVQ_APP(64, KVQ_INT8_ASYM);
    else if (fmt_static(fmt)) e = KVQ_APP(64, KVQ_INT8_CHANNEL);
    else e = KVQ_APP(64, KVQ_BF16);
  }
#undef KVQ_APP
  return int(e);
}

int launch_decode_partial(const void* q, int32_t B, const void* kc, const void* vc,
                          const void* ks, const void* vs, const int32_t* tables,
                          const int32_t* ctx, int32_t max_ctx, float sm_scale,
                          const DecodePlan& plan, void* ws, kvq_fmt fmt, const kvq_dims& d,
                          void* stream, int n_query) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int G = d.n_q_heads / d.n_kv_heads;
  cudaError_t e;
#define KVQ_DEC(DD, FF) decode_dispatch2<DD, FF>(G, q, B, kc, vc, ks, vs, tables, ctx, max_ctx, sm_scale, plan, ws, d, pt, n_query, st)
  const int pt = fmt == KVQ_INT8_TENSOR;
  if (d.head_dim == 128) {
    if (fmt == KVQ_FP8_E4M3) e = KVQ_DEC(128, KVQ_FP8_E4M3);
    else if (fmt == KVQ_FP8_E5M2) e = KVQ_DEC(128, KVQ_FP8_E5M2);
    else if (fmt == KVQ_INT8_ASYM) e = KVQ_DEC(128, KVQ_INT8_ASYM);
    else if (fmt_static(fmt)) e = KVQ_DEC(128, KVQ_INT8_CHANNEL);
    else e = KVQ_DEC(128, KVQ_BF16);
  } else {
    if (fmt == KVQ_FP8_E4M3) e = KVQ_DEC(64, KVQ_FP8_E4M3);
    else if (fmt == KVQ_FP8_E5M2) e = KVQ_DEC(64, KVQ_FP8_E5M2);
    else if (fmt == KVQ_INT8_ASYM) e = KVQ_DEC(64, KVQ_INT8_ASYM);
    else if (fmt_static(fmt)) e = KVQ_DEC(64, KVQ_INT8_CHANNEL);
    else e = KVQ_DEC(64, KVQ_BF16);
  }
#undef KVQ_DEC
  return int(e);
}

int launch_decode_merge(int32_t B, const int32_t* ctx, int32_t max_ctx, void* out, bool out_f32,
                        const void* ws, const DecodePlan& plan, const kvq_dims& d, void* stream,
                        int rows_per_count) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const float* po = static_cast<const float*>(ws);
  const float* pml = reinterpret_cast<const float*>(static_cast<const char*>(ws) + plan.o_bytes);
  const int32_t* pcnt =
      reinterpret_cast<const int32_t*>(static_cast<const char*>(ws) + plan.o_bytes + plan.ml_bytes);
  const int rows = int(int64_t(B) * d.n_q_heads);
  const dim3 grid(unsigned((rows + 3) / 4));
  // G: query rows per row group, the unit part_cnt is kept for
  const int W = d.max_blocks_per_seq, Hq = d.n_q_heads;
  int G = rows_per_count;
  if (G <= 0) row_groups(d.n_q_heads / d.n_kv_heads, &G);
  cudaError_t e;
  if (d.head_dim == 128) {
    if (out_f32)
      e = launch_pdl(merge_kernel<128, float>, grid, dim3(128), 0, st, ctx, Hq, G, plan.slots,
                     max_ctx, W, po, pml, pcnt, static_cast<float*>(out), rows);
    else
      e = launch_pdl(merge_kernel<128, __nv_bfloat16>, grid, dim3(128), 0, st, ctx, Hq, G,
                     plan.slots, max_ctx, W, po, pml, pcnt, static_cast<__nv_bfloat16*>(out), rows);
  } else {
    if (out_f32)
      e = launch_pdl(merge_kernel<64, float>, grid, dim3(128), 0, st, ctx, Hq, G, plan.slots,
                     max_ctx, W, po, pml, pcnt, static_cast<float*>(out), rows);
    else
      e = launch_pdl(merge_kernel<64, __nv_bfloat16>, grid, dim3(128), 0, st, ctx, Hq, G,
                     plan.slots, max_ctx, W, po, pml, pcnt, static_cast<__nv_bfloat16*>(out), rows);
  }
  if (e != cudaSuccess) return int(e);
  return int(cudaGetLastError());
}

namespace {
template <int D, int G, int BITS>
cudaError_t kivi_dispatch3(const void* q, int32_t B, const void* kc, const void* vc, const void* km,
                           const void* vm, const int32_t* tables, const int32_t* lens,
                           int32_t max_len, float sm_scale, const DecodePlan& plan, void* ws,
                           const kvq_dims& d, cudaStream_t st) {
  using C = KiviCfg<D, G, BITS>;
  auto kern = decode_kivi_kernel<D, G, BITS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                           int(cudaSharedmemCarveoutMaxShared));
  if (e != cudaSuccess) return e;
  int dev = 0, smem_sm = 0, reserved = 0;
  e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev);
  if (e != cudaSuccess) return e;
  const int per_sm = std::max(1, std::min(2, smem_sm / (C::SMEM + reserved)));
  float* po = static_cast<float*>(ws);
  float* pml = reinterpret_cast<float*>(static_cast<char*>(ws) + plan.o_bytes);
  int32_t* pcnt = reinterpret_cast<int32_t*>(static_cast<char*>(ws) + plan.o_bytes + plan.ml_bytes);
  const int64_t grid = int64_t(device_sm_count()) * per_sm;
  kern<<<dim3(unsigned(grid)), 256, C::SMEM, st>>>(
      static_cast<const __nv_bfloat16*>(q), static_cast<const uint8_t*>(kc),
      static_cast<const uint8_t*>(vc), static_cast<const __nv_bfloat16*>(km),
      static_cast<const __nv_bfloat16*>(vm), tables, lens, B, d.n_kv_heads, d.num_blocks,
      d.max_blocks_per_seq, max_len, plan.partition / kTileTokens, plan.slots, sm_scale * kLog2e,
      decode_wait_limit(), po, pml, pcnt);
  return cudaGetLastError();
}

template <int D, int BITS>
cudaError_t kivi_dispatch2(int G, const void* q, int32_t B, const void* kc, const void* vc,
                           const void* km, const void* vm, const int32_t* tables,
                           const int32_t* lens, int32_t max_len, float sm_scale,
                           const DecodePlan& plan, void* ws, const kvq_dims& d, cudaStream_t st) {
  switch (G) {
    case 1: return kivi_dispatch3<D, 1, BITS>(q, B, kc, vc, km, vm, tables, lens, max_len, sm_scale, plan, ws, d, st);
    case 2: return kivi_dispatch3<D, 2, BITS>(q, B, kc, vc, km, vm, tables, lens, max_len, sm_scale, plan, ws, d, st);
    case 4: return kivi_dispatch3<D, 4, BITS>(q, B, kc, vc, km, vm, tables, lens, max_len, sm_scale, plan, ws, d, st);
    default: return kivi_dispatch3<D, 8, BITS>(q, B, kc, vc, km, vm, tables, lens, max_len, sm_scale, plan, ws, d, st);
  }
}
}  // namespace

int launch_kivi_decode(const void* q, int32_t B, const void* kc, const void* vc, const void* km,
                       const void* vm, const int32_t* tables, const int32_t* qlens,
                       int32_t max_qlen, const void* rk, const void* rv,
                       const int32_t* rtables, const int32_t* rlens, int32_t max_rlen,
                       float sm_scale, void* out, bool out_f32, void* ws, const DecodePlan& pa,
                       const DecodePlan& pb, int bits, const kvq_dims& d, const kvq_dims& rd,
                       void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int G = d.n_q_heads / d.n_kv_heads;
  void* ws_b = static_cast<char*>(ws) + pa.total;
  cudaError_t e;
  // the quantized groups
  if (d.head_dim == 128)
    e = bits == 2 ? kivi_dispatch2<128, 2>(G, q, B, kc, vc, km, vm, tables, qlens, max_qlen, sm_scale, pa, ws, d, st)
                  : kivi_dispatch2<128, 4>(G, q, B, kc, vc, km, vm, tables, qlens, max_qlen, sm_scale, pa, ws, d, st);
  else
    e = bits == 2 ? kivi_dispatch2<64, 2>(G, q, B, kc, vc, km, vm, tables, qlens, max_qlen, sm_scale, pa, ws, d, st)
                  : kivi_dispatch2<64, 4>(G, q, B, kc, vc, km, vm, tables, qlens, max_qlen, sm_scale, pa, ws, d, st);
  if (e != cudaSuccess) return int(e);
  // the residual tokens and the merge, one CTA per (sequence, KV head),
  // launched as a programmatic dependent of the groups kernel
  (void)pb;
  const float* poa = static_cast<const float*>(ws);
  const float* pmla = reinterpret_cast<const float*>(static_cast<const char*>(ws) + pa.o_bytes);
  const int32_t* pca = reinterpret_cast<const int32_t*>(static_cast<const char*>(ws) + pa.o_bytes + pa.ml_bytes);
  const dim3 grid(unsigned(int64_t(B) * d.n_kv_heads));
  const float qk = sm_scale * kLog2e;
  auto go = [&](auto kern, auto* o) {
    return launch_pdl(kern, grid, dim3(128), 0, st, static_cast<const __nv_bfloat16*>(q), d.n_kv_heads,
                      qlens, pa.slots, max_qlen, d.max_blocks_per_seq, poa, pmla, pca,
                      static_cast<const __nv_bfloat16*>(rk), static_cast<const __nv_bfloat16*>(rv), rtables,
                      rlens, rd.num_blocks, rd.max_blocks_per_seq, max_rlen, qk, o);
  };
#define KVQ_RM(DD, GG)                                                                        \
  e = out_f32 ? go(kivi_residual_merge_kernel<DD, GG, float>, static_cast<float*>(out))       \
              : go(kivi_residual_merge_kernel<DD, GG, __nv_bfloat16>, static_cast<__nv_bfloat16*>(out))
#define KVQ_RM_G(DD)        \
  switch (G) {              \
    case 1: KVQ_RM(DD, 1); break; \
    case 2: KVQ_RM(DD, 2); break; \
    case 4: KVQ_RM(DD, 4); break; \
    default: KVQ_RM(DD, 8); break; \
  }
  if (d.head_dim == 128) {
    KVQ_RM_G(128)
  } else {
    KVQ_RM_G(64)
  }
#undef KVQ_RM_G
#undef KVQ_RM
  if (e != cudaSuccess) return int(e);
  return int(cudaGetLastError());
}

int read_device_error(uint32_t* flags, int clear) {
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return int(e);
  unsigned int v = 0;
  e = cudaMemcpyFromSymbol(&v, g_error_word, sizeof(v));
  if (e != cudaSuccess) return int(e);
  *flags = v;
  if (clear && v) {
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero));
    if (e != cudaSuccess) return int(e);
  }
  return 0;
}

}  // namespace kvq

// KIVI-style low-bit KV cache for sm_100a: keys quantized per channel over
// groups of 128 positions, values per token, b = 2 or 4 bits, asymmetric
// (scale, minimum) in BF16; the positions after the last complete group stay
// in full precision in a BF16 cache of their own.
//
// Sources (web pages, by title and section):
//  "KV Cache compression" - "2.1" (K has outlier channels, V a per-token
//     distribution: quantize K per channel and V per token) and "3.1", KIVI
//     (asymmetric 2-bit codes, K per channel, V per token, the most recent
//     tokens kept in full precision as a residual, no tuning).
//  "KV cache quantization: what FP8/INT8 K and V really give" - "Formats you
//     will actually meet" (the mixed-precision 4-bit variants quantize K per
//     channel and V per token) and the opening paragraph (4-bit storage is a
//     quarter of BF16).
//
// This header holds the group quantizer (kvq_kivi_append). Included by
// kvq_kernels.cu (it uses the error word defined there).
#pragma once

namespace kvq {
namespace kivi {

// 16 codes of b bits -> their packed form (2b bytes), in the order the decode
// kernel expands with one shift and one mask per 4 output bytes: code e = 4m +
// j sits at bit 8j + b*m of packed word m / (4 / b) (b = 2: one word; b = 4:
// word m / 2, bit 8j + 4 (m % 2)).
template <int BITS>
__device__ __forceinline__ void pack16(const uint8_t (&c)[16], uint32_t (&w)[BITS / 2]) {
#pragma unroll
  for (int i = 0; i < BITS / 2; ++i) w[i] = 0u;
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const int m = e >> 2, j = e & 3;
    if constexpr (BITS == 2) w[0] |= uint32_t(c[e]) << (8 * j + 2 * m);
    else w[m >> 1] |= uint32_t(c[e]) << (8 * j + 4 * (m & 1));
  }
}

// code = clamp(rint(RN(x - z) / s), 0, 2^b - 1), IEEE f32 subtraction and
// division; a zero scale gives 0
template <int BITS>
__device__ __forceinline__ uint8_t code_of(float x, float s, float z) {
  if (!(s > 0.f)) return 0;
  const float q = __fdiv_rn(__fsub_rn(x, z), s);
  const int c = __float2int_rn(fminf(fmaxf(q, -1.f), float((1 << BITS) + 1)));
  return uint8_t(min((1 << BITS) - 1, max(0, c)));
}

// (s, z) of a group from its float minimum and maximum: z = bf16(min),
// s = bf16(f32(max - min) / (2^b - 1)); a zero minimum or range is +0
template <int BITS>
__device__ __forceinline__ void params(float lo, float hi, __nv_bfloat16& s, __nv_bfloat16& z) {
  const float span = __fsub_rn(hi, lo);
  z = __float2bfloat16_rn(lo == 0.f ? 0.f : lo);
  const float sv = span == 0.f ? 0.f : __fdiv_rn(span, float((1 << BITS) - 1));
  s = __float2bfloat16_rn(sv);
}

// Byte offset, in a packed K page, of the 2b-byte unit of (token t, 16-channel
// chunk c): the page is [token group t/8][chunk c][token t%8][2b bytes], the
// tensor-core K operand layout with every 16-byte row packed to 2b bytes.
template <int D, int BITS>
__device__ __forceinline__ int k_unit(int t, int c) {
  return (((t >> 3) * (D / 16) + c) * 8 + (t & 7)) * (2 * BITS);
}

// One CTA per (group of 128 tokens of the call, KV head, K or V).
//  K (blockIdx.z == 0): the group's K rows staged in shared memory; per
//    channel the minimum and maximum over the 128 positions give its (s, z);
//    every (token, 16-channel chunk) is coded and packed into the group's eight
//    pages; page i of the group stores the (s, z) of channels [i D/8, (i+1) D/8).
//  V (blockIdx.z == 1): per token its minimum and maximum over the D channels
//    give its (s, z), stored with the token; the codes are staged and each
//    (page, channel) packs its 16 tokens (the V page is stored transposed).
// The group's 128 slots must fill eight pages in order (slot % 16 == token %
// 16, one block per 16 tokens); a group that does not is skipped and flagged
// (KVQ_DEVERR_SLOT), a group of negative slots is skipped.
template <int D, int BITS>
__global__ void __launch_bounds__(256) kivi_append_kernel(
    const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
    const int64_t* __restrict__ slots, int Hk, int NB, uint8_t* __restrict__ kc,
    uint8_t* __restrict__ vc, __nv_bfloat16* __restrict__ kmeta, __nv_bfloat16* __restrict__ vmeta) {
  constexpr int PPAGE = kBlockSize * D * BITS / 8;     // packed page bytes
  constexpr int ROWP = D + 8;                          // staged row (bf16 elements), padded
  // the staged rows; the V pass overwrites each row with its codes (bytes)
  __shared__ __align__(16) __nv_bfloat16 xs[128 * ROWP];
  __shared__ int64_t sls[128], blk[8];
  __shared__ float red[2][2][D];
  __shared__ __nv_bfloat16 ps[D], pz[D];

  const int g = blockIdx.x, h = blockIdx.y, isv = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t t0 = int64_t(g) * 128;
  const int64_t nslots = int64_t(NB) * kBlockSize;
  const __nv_bfloat16* src = isv ? v : k;
  // stage the 128 rows (16-byte loads)
  for (int u = tid; u < 128 * D / 8; u += blockDim.x) {
    const int t = u / (D / 8), c8 = u % (D / 8);
    *reinterpret_cast<uint4*>(xs + t * ROWP + c8 * 8) =
        *reinterpret_cast<const uint4*>(src + ((t0 + t) * Hk + h) * D + c8 * 8);
  }
  if (tid < 128) sls[tid] = slots[t0 + tid];
  __syncthreads();
  bool neg = true, good = true;
  if (tid < 128) {
    const int64_t sl = sls[tid];
    neg = sl < 0;
    good = sl >= 0 && sl < nslots && int(sl % kBlockSize) == (tid & 15) &&
           sl / kBlockSize == sls[tid & ~15] / kBlockSize;
  }
  const int all_neg = __syncthreads_and(neg);
  const int all_good = __syncthreads_and(good);
  if (all_neg) return;                                   // a skipped group
  if (!all_good) {                                       // out of range or out of order
    if (tid == 0) flag_error(KVQ_DEVERR_SLOT);
    return;
  }
  if (tid < 8) blk[tid] = sls[16 * tid] / kBlockSize;
  __syncthreads();

  if (!isv) {
    // ---- K: per-channel range over the 128 positions
    {
      const int d = tid % D, part = tid / D, nparts = 256 / D;   // 2 (D=128) or 4 (D=64)
      float lo = INFINITY, hi = -INFINITY;
      for (int t = part; t < 128; t += nparts) {
        const float x = __bfloat162float(xs[t * ROWP + d]);
        lo = fminf(lo, x);
        hi = fmaxf(hi, x);
      }
      if (part < 2) { red[0][part][d] = lo; red[1][part][d] = hi; }
      __syncthreads();
      if (nparts == 4 && part >= 2) {
        red[0][part - 2][d] = fminf(red[0][part - 2][d], lo);
        red[1][part - 2][d] = fmaxf(red[1][part - 2][d], hi);
      }
      __syncthreads();
      if (tid < D) {
        __nv_bfloat16 s, z;
        params<BITS>(fminf(red[0][0][tid], red[0][1][tid]), fmaxf(red[1][0][tid], red[1][1][tid]), s, z);
        ps[tid] = s;
        pz[tid] = z;
        // page i of the group holds channels [i D/8, (i+1) D/8)
        constexpr int CPP = D / 8;
        const int pg = tid / CPP, j = tid % CPP;
        __nv_bfloat16* m = kmeta + ((blk[pg] * Hk + h) * kBlockSize + j) * 2;
        m[0] = s;
        m[1] = z;
      }
      __syncthreads();
    }
    // ---- codes: one (token, 16-channel chunk) per unit
    for (int u = tid; u < 128 * (D / 16); u += blockDim.x) {
      const int t = u / (D / 16), c = u % (D / 16);
      uint8_t code[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int d = c * 16 + e;
        code[e] = code_of<BITS>(__bfloat162float(xs[t * ROWP + d]), __bfloat162float(ps[d]),
                                __bfloat162float(pz[d]));
      }
      uint32_t w[BITS / 2];
      pack16<BITS>(code, w);
      uint8_t* dst = kc + (blk[t >> 4] * Hk + h) * PPAGE + k_unit<D, BITS>(t & 15, c);
      if constexpr (BITS == 2) *reinterpret_cast<uint32_t*>(dst) = w[0];
      else *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
    }
  } else {
    // ---- V: per-token range over the D channels, one warp per token
    for (int t = warp; t < 128; t += 8) {
      float lo = INFINITY, hi = -INFINITY;
#pragma unroll
      for (int i = 0; i < D / 32; ++i) {
        const float x = __bfloat162float(xs[t * ROWP + lane + 32 * i]);
        lo = fminf(lo, x);
        hi = fmaxf(hi, x);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
        hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
      }
      __nv_bfloat16 s, z;
      params<BITS>(lo, hi, s, z);
      const float sf = __bfloat162float(s), zf = __bfloat162float(z);
      uint8_t cv[D / 32];
#pragma unroll
      for (int i = 0; i < D / 32; ++i)
        cv[i] = code_of<BITS>(__bfloat162float(xs[t * ROWP + lane + 32 * i]), sf, zf);
      __syncwarp();                                      // the row is read: codes over it
      uint8_t* crow = reinterpret_cast<uint8_t*>(xs + t * ROWP);
#pragma unroll
      for (int i = 0; i < D / 32; ++i) crow[lane + 32 * i] = cv[i];
      if (lane == 0) {
        __nv_bfloat16* m = vmeta + ((blk[t >> 4] * Hk + h) * kBlockSize + (t & 15)) * 2;
        m[0] = s;
        m[1] = z;
      }
    }
    __syncthreads();
    // ---- pack: one (page, channel) per unit, its 16 tokens
    for (int u = tid; u < 8 * D; u += blockDim.x) {
      const int pg = u / D, d = u % D;
      uint8_t code[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) code[e] = reinterpret_cast<const uint8_t*>(xs + (pg * 16 + e) * ROWP)[d];
      uint32_t w[BITS / 2];
      pack16<BITS>(code, w);
      uint8_t* dst = vc + (blk[pg] * Hk + h) * PPAGE + d * (2 * BITS);
      if constexpr (BITS == 2) *reinterpret_cast<uint32_t*>(dst) = w[0];
      else *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
    }
  }
}

}  // namespace kivi

int launch_kivi_append(const void* k, const void* v, const int64_t* slots, int32_t T, void* kc,
                       void* vc, void* km, void* vm, int bits, const kvq_dims& d, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const dim3 grid(unsigned(T / 128), unsigned(d.n_kv_heads), 2);
  auto K = static_cast<const __nv_bfloat16*>(k);
  auto V = static_cast<const __nv_bfloat16*>(v);
  auto kcp = static_cast<uint8_t*>(kc);
  auto vcp = static_cast<uint8_t*>(vc);
  auto kmp = static_cast<__nv_bfloat16*>(km);
  auto vmp = static_cast<__nv_bfloat16*>(vm);
  if (d.head_dim == 128) {
    if (bits == 2) kivi::kivi_append_kernel<128, 2><<<grid, 256, 0, st>>>(K, V, slots, d.n_kv_heads, d.num_blocks, kcp, vcp, kmp, vmp);
    else kivi::kivi_append_kernel<128, 4><<<grid, 256, 0, st>>>(K, V, slots, d.n_kv_heads, d.num_blocks, kcp, vcp, kmp, vmp);
  } else {
    if (bits == 2) kivi::kivi_append_kernel<64, 2><<<grid, 256, 0, st>>>(K, V, slots, d.n_kv_heads, d.num_blocks, kcp, vcp, kmp, vmp);
    else kivi::kivi_append_kernel<64, 4><<<grid, 256, 0, st>>>(K, V, slots, d.n_kv_heads, d.num_blocks, kcp, vcp, kmp, vmp);
  }
  return int(cudaGetLastError());
}

}  // namespace kvq

// Log-sum-exp merge of the decode kernels' split-K partials into the output
// rows: one set (kvq_decode_merge) or two sets of the same rows (the KIVI-style
// cache's quantized groups and its BF16 residual). Included by kvq_kernels.cu.
#pragma once

namespace kvq {

// ------------------------------------------------------------------ merge
// One warp per (sequence, query row), four rows per CTA: combine the chunk
// partials (m_i, l_i, o_i) as m = max m_i, l = sum l_i 2^(m_i - m),
// o = sum o_i 2^(m_i - m) / l. Lane i holds slot i's (m, l) (32 slots at a
// time); each lane owns D/32 consecutive channels and reads them as one vector
// per slot, so a row's partials stream in with every load in flight.
template <int D>
struct MergeVec {
  static constexpr int N = D / 32;
  float v[N];
  __device__ __forceinline__ void load(const float* p) {
    if constexpr (N == 4) {
      const float4 x = *reinterpret_cast<const float4*>(p);
      v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
    } else {
      const float2 x = *reinterpret_cast<const float2*>(p);
      v[0] = x.x; v[1] = x.y;
    }
  }
};

template <int D, typename OutT>
__global__ void __launch_bounds__(128) merge_kernel(const int32_t* __restrict__ ctx_lens, int Hq,
                                                    int G, int slots, int max_ctx, int W,
                                                    const float* __restrict__ part_o,
                                                    const float* __restrict__ part_ml,
                                                    const int32_t* __restrict__ part_cnt,
                                                    OutT* __restrict__ out, int rows) {
  constexpr int N = D / 32;
  constexpr int PRE = 8;                                   // slots whose vectors load up front
  const int lane = threadIdx.x & 31;
  const int bq = blockIdx.x * 4 + (threadIdx.x >> 5);      // b * Hq + row
  tc::grid_dep_wait();                                     // the partials are complete
  if (bq >= rows) return;
  const int b = bq / Hq;
  const int64_t r0 = int64_t(bq) * slots;
  // The length, the count, the first 32 slots' (m, l) and the first PRE slots'
  // vectors are requested together, before the count is known (every slot
  // index below `slots` lies inside the workspace; values of slots past the
  // count are never used), so a row costs one round trip to memory.
  const int ctx_raw = ctx_lens[b];
  const int cnt_raw = part_cnt[bq / G];
  float2 ml = make_float2(-INFINITY, 0.f);
  if (lane < slots) ml = *reinterpret_cast<const float2*>(part_ml + (r0 + lane) * 2);
  MergeVec<D> x[PRE];
#pragma unroll
  for (int j = 0; j < PRE; ++j)
    if (j < slots) x[j].load(part_o + (r0 + j) * D + lane * N);
  int ctx = ctx_raw;
  if (ctx < 0 || ctx > max_ctx || int64_t(ctx) > int64_t(W) * kBlockSize) ctx = 0;
  // partials written for this (sequence, row group) by the decode kernel
  const int n = ctx > 0 ? min(slots, max(0, cnt_raw)) : 0;
  if (lane >= n) ml = make_float2(-INFINITY, 0.f);
  float M = ml.x;
  for (int s0 = 32; s0 < n; s0 += 32)
    if (s0 + lane < n) M = fmaxf(M, part_ml[(r0 + s0 + lane) * 2]);
  M = warp_max(M);
  float o[N], l = 0.f;
#pragma unroll
  for (int i = 0; i < N; ++i) o[i] = 0.f;
  if (M != -INFINITY) {
    // the sums run over the slots in order, as a single thread per channel would
    const float fl0 = exp2f(ml.x - M);
#pragma unroll
    for (int j = 0; j < PRE; ++j) {
      if (j >= n) break;
      const float f = __shfl_sync(0xffffffffu, fl0, j);
      const float ls = __shfl_sync(0xffffffffu, ml.y, j);
      l += ls * f;
#pragma unroll
      for (int i = 0; i < N; ++i) o[i] += x[j].v[i] * f;
    }
    for (int s0 = 0; s0 < n; s0 += 32) {
      float2 mls = ml;
      float fl = fl0;
      if (s0 > 0) {
        mls = make_float2(-INFINITY, 0.f);
        if (s0 + lane < n) mls = *reinterpret_cast<const float2*>(part_ml + (r0 + s0 + lane) * 2);
        fl = exp2f(mls.x - M);
      }
      const int cnt = min(32, n - s0);
      // slots past the first PRE: eight slots' vectors are requested before any is summed
      for (int s8 = (s0 == 0 ? PRE : 0); s8 < cnt; s8 += 8) {
        MergeVec<D> y[8];
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (s8 + j < cnt) y[j].load(part_o + (r0 + s0 + s8 + j) * D + lane * N);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (s8 + j >= cnt) break;
          const float f = __shfl_sync(0xffffffffu, fl, s8 + j);
          const float ls = __shfl_sync(0xffffffffu, mls.y, s8 + j);
          l += ls * f;
#pragma unroll
          for (int i = 0; i < N; ++i) o[i] += y[j].v[i] * f;
        }
      }
    }
  }
  // l == 0: nothing attended (zeros); a NaN l (a piece that timed out wrote
  // NaN markers) gives NaN
  float r[N];
#pragma unroll
  for (int i = 0; i < N; ++i) r[i] = l != 0.f ? o[i] / l : 0.f;
  OutT* dst = out + int64_t(bq) * D + lane * N;
  if constexpr (sizeof(OutT) == 4) {
    if constexpr (N == 4) *reinterpret_cast<float4*>(dst) = make_float4(r[0], r[1], r[2], r[3]);
    else *reinterpret_cast<float2*>(dst) = make_float2(r[0], r[1]);
  } else {
    if constexpr (N == 4) {
      const __nv_bfloat162 a0 = __floats2bfloat162_rn(r[0], r[1]), a1 = __floats2bfloat162_rn(r[2], r[3]);
      *reinterpret_cast<uint2*>(dst) = make_uint2(*reinterpret_cast<const uint32_t*>(&a0),
                                                  *reinterpret_cast<const uint32_t*>(&a1));
    } else {
      *reinterpret_cast<__nv_bfloat162*>(dst) = __floats2bfloat162_rn(r[0], r[1]);
    }
  }
}

// Merge of two partial sets of the same rows: the quantized groups' partials
// (a) and the residual tokens' (b), each with its own context lengths, slot
// count and per-(sequence, row group) counts.
template <int D, typename OutT>
__global__ void __launch_bounds__(128) merge2_kernel(
    int Hq, int G, const int32_t* __restrict__ ctx_a, int slots_a, int max_a, int W_a,
    const float* __restrict__ po_a, const float* __restrict__ pml_a, const int32_t* __restrict__ pc_a,
    const int32_t* __restrict__ ctx_b, int slots_b, int max_b, int W_b,
    const float* __restrict__ po_b, const float* __restrict__ pml_b, const int32_t* __restrict__ pc_b,
    int group_mask_a, OutT* __restrict__ out) {
  const int bq = blockIdx.x;
  const int b = bq / Hq;
  const int d = threadIdx.x;
  int ca = ctx_a[b], cb = ctx_b[b];
  if (ca < 0 || ca > max_a || int64_t(ca) > int64_t(W_a) * kBlockSize) ca = 0;
  ca &= group_mask_a;
  if (cb < 0 || cb > max_b || int64_t(cb) > int64_t(W_b) * kBlockSize) cb = 0;
  const int na = ca > 0 ? min(slots_a, max(0, pc_a[bq / G])) : 0;
  const int nb = cb > 0 ? min(slots_b, max(0, pc_b[bq / G])) : 0;
  const int64_t ra = int64_t(bq) * slots_a, rb = int64_t(bq) * slots_b;
  float M = -INFINITY;
  for (int s = 0; s < na; ++s) M = fmaxf(M, pml_a[(ra + s) * 2]);
  for (int s = 0; s < nb; ++s) M = fmaxf(M, pml_b[(rb + s) * 2]);
  float o = 0.f, l = 0.f;
  if (M != -INFINITY) {
    for (int s = 0; s < na; ++s) {
      const float f = exp2f(pml_a[(ra + s) * 2] - M);
      l += pml_a[(ra + s) * 2 + 1] * f;
      o += po_a[(ra + s) * D + d] * f;
    }
    for (int s = 0; s < nb; ++s) {
      const float f = exp2f(pml_b[(rb + s) * 2] - M);
      l += pml_b[(rb + s) * 2 + 1] * f;
      o += po_b[(rb + s) * D + d] * f;
    }
  }
  const float r = l != 0.f ? o / l : 0.f;            // NaN l (a timed-out piece): NaN
  if constexpr (sizeof(OutT) == 4) out[int64_t(bq) * D + d] = r;
  else out[int64_t(bq) * D + d] = __float2bfloat16_rn(r);
}

}  // namespace kvq

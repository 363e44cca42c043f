// Log-sum-exp merge of the decode kernels' split-K partials into the output
// rows (kvq_decode_merge), and the KIVI-style cache's BF16 residual attention
// fused with the merge of its quantized groups' partials. Included by
// kvq_kernels.cu.
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

// ------------------------------------------------------- KIVI residual
// The KIVI-style decode's second half: the BF16 residual tokens (those after
// the last complete group) of one (sequence, KV head), attended in FP32 on the
// CUDA cores, then the log-sum-exp merge with the quantized groups' partial
// slots of the same rows. One CTA of 128 threads per (sequence, KV head)
// covers the group's G query rows:
//   scores   thread t takes token t of each 128-token chunk: its K row from
//            the BF16 operand page (16-byte chunks 128 bytes apart), dot
//            products with the G query rows (times sm_scale log2 e) held in
//            shared memory;
//   values   thread d < D accumulates O[g][d] over the chunk's tokens from the
//            transposed V page: one 16-byte load per 8 tokens of its channel;
//   softmax  online over the chunks in base 2, as the decode kernels do;
//   merge    m = max(m_res, m_i), l and o summed with weights 2^(m_x - m).
// Launched as a programmatic dependent of the groups kernel, which does not
// signal early: the launch overlaps the groups kernel's end, and the
// partials are read after the grid dependency wait, through plain pointers
// and L2-coherent loads (never taken as invariant data that could be read
// ahead of the wait).
template <int D, int G, typename OutT>
__global__ void __launch_bounds__(128) kivi_residual_merge_kernel(
    const __nv_bfloat16* __restrict__ q, int Hk, const int32_t* ctx_a, int slots_a, int max_a,
    int W_a, const float* po_a, const float* pml_a, const int32_t* pc_a,
    const __nv_bfloat16* __restrict__ rk,
    const __nv_bfloat16* __restrict__ rv, const int32_t* __restrict__ rtables,
    const int32_t* __restrict__ rlens, int NBr, int Wr, int max_r, float qk_scale,
    OutT* __restrict__ out) {
  using namespace tc;
  __shared__ __align__(16) float qsh[G][D];
  __shared__ __align__(16) float psh[128][G];
  __shared__ float red[4][G];
  const int b = blockIdx.x / Hk, h = blockIdx.x % Hk;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int Hq = Hk * G;
  const int64_t row0 = int64_t(b) * Hq + int64_t(h) * G;        // first query row of the group
  int rl = rlens[b];
  if (rl < 0 || rl > max_r || int64_t(rl) > int64_t(Wr) * kBlockSize) {
    if (h == 0 && tid == 0) flag_error(KVQ_DEVERR_CONTEXT);
    rl = 0;
  }
  for (int i = tid; i < G * D; i += 128) qsh[i / D][i % D] = qk_scale * __bfloat162float(q[row0 * D + i]);
  __syncthreads();

  constexpr int64_t PAGE = int64_t(kBlockSize) * D * 2;           // bytes of one BF16 page
  const uint8_t* rkb = reinterpret_cast<const uint8_t*>(rk);
  const uint8_t* rvb = reinterpret_cast<const uint8_t*>(rv);
  auto unpack8 = [](const uint4& u, float (&f)[8]) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  };
  float m[G], lsum[G], o[G];
#pragma unroll
  for (int g = 0; g < G; ++g) { m[g] = -INFINITY; lsum[g] = 0.f; o[g] = 0.f; }
  for (int t0 = 0; t0 < rl; t0 += 128) {
    // ---- scores of token t0 + tid
    const int t = t0 + tid;
    float s[G];
#pragma unroll
    for (int g = 0; g < G; ++g) s[g] = -INFINITY;
    if (t < rl) {
      const int blk = rtables[int64_t(b) * Wr + t / kBlockSize];
      if (blk < 0 || blk >= NBr) {
        flag_error(KVQ_DEVERR_BLOCK);
      } else {
        const int tt = t % kBlockSize;
        const uint8_t* krow = rkb + (int64_t(blk) * Hk + h) * PAGE + (tt / 8) * 8 * D * 2 + (tt % 8) * 16;
        float acc[G];
#pragma unroll
        for (int g = 0; g < G; ++g) acc[g] = 0.f;
#pragma unroll 4
        for (int c = 0; c < D / 8; ++c) {
          float kf[8];
          unpack8(*reinterpret_cast<const uint4*>(krow + c * 128), kf);
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const float4 qa = *reinterpret_cast<const float4*>(&qsh[g][c * 8]);
            const float4 qb = *reinterpret_cast<const float4*>(&qsh[g][c * 8 + 4]);
            acc[g] = fmaf(qa.x, kf[0], acc[g]); acc[g] = fmaf(qa.y, kf[1], acc[g]);
            acc[g] = fmaf(qa.z, kf[2], acc[g]); acc[g] = fmaf(qa.w, kf[3], acc[g]);
            acc[g] = fmaf(qb.x, kf[4], acc[g]); acc[g] = fmaf(qb.y, kf[5], acc[g]);
            acc[g] = fmaf(qb.z, kf[6], acc[g]); acc[g] = fmaf(qb.w, kf[7], acc[g]);
          }
        }
#pragma unroll
        for (int g = 0; g < G; ++g) s[g] = acc[g];
      }
    }
    // ---- the chunk's maxima, the new references, the weights
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float wm = warp_max_f32(s[g]);
      if (lane == 0) red[warp][g] = wm;
    }
    __syncthreads();
    float alpha[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float cm = fmaxf(fmaxf(red[0][g], red[1][g]), fmaxf(red[2][g], red[3][g]));
      const float mn = fmaxf(m[g], cm);
      const float a = exp2f(m[g] - mn);
      alpha[g] = (mn == m[g] || mn == -INFINITY) ? 1.f : a;
      m[g] = mn;
      const float e2 = exp2f(s[g] - mn);
      const float p = s[g] != -INFINITY ? e2 : 0.f;
      psh[tid][g] = p;
      lsum[g] = lsum[g] * alpha[g] + p;
      o[g] *= alpha[g];
    }
    __syncthreads();
    // ---- values: channel tid, the chunk's tokens 8 at a time (a page holds
    // two 8-token halves; t0 is a multiple of 128, so no half straddles pages)
    if (tid < D) {
      const int nt = min(128, rl - t0);
      for (int u = 0; u < nt; u += 8) {
        const int tu = t0 + u;
        const int blk = rtables[int64_t(b) * Wr + tu / kBlockSize];
        if (blk < 0 || blk >= NBr) continue;                      // its weights are 0
        float vf[8];
        unpack8(*reinterpret_cast<const uint4*>(rvb + (int64_t(blk) * Hk + h) * PAGE +
                                                (int64_t((tu % kBlockSize) / 8) * D + tid) * 16), vf);
        const int ne = min(8, nt - u);                            // tokens past the end: not read
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          if (e < ne) {
#pragma unroll
            for (int g = 0; g < G; ++g) o[g] = fmaf(psh[u + e][g], vf[e], o[g]);
          }
        }
      }
    }
    __syncthreads();                                              // psh and red are rewritten
  }
  // ---- the residual's sums
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const float ws = warp_sum(lsum[g]);
    if (lane == 0) red[warp][g] = ws;
  }
  __syncthreads();
  float lres[G];
#pragma unroll
  for (int g = 0; g < G; ++g) lres[g] = red[0][g] + red[1][g] + red[2][g] + red[3][g];

  // ---- merge with the groups' partials (written by the preceding kernel),
  // eight slots at a time: the slots' (m, l) of all G rows are loaded by one
  // thread each into shared memory while every channel thread requests its
  // G x 8 partial values, so a chunk costs one round trip to memory
  grid_dep_wait();
  int ca = __ldcg(ctx_a + b);
  if (ca < 0 || ca > max_a || int64_t(ca) > int64_t(W_a) * kBlockSize) ca = 0;
  ca &= ~127;
  const int na = ca > 0 ? min(slots_a, max(0, __ldcg(pc_a + int64_t(b) * Hk + h))) : 0;
  __shared__ float2 mls[G][8];
  float M[G], ll[G], oo[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    M[g] = m[g];                                                // the residual's (or -inf)
    ll[g] = lres[g];
    oo[g] = o[g];
  }
  for (int s0 = 0; s0 < na; s0 += 8) {
    const int ns = min(8, na - s0);
    __syncthreads();                                            // the previous chunk's mls are used
    if (tid < G * 8) {
      const int g = tid >> 3, j = tid & 7;
      float2 v = make_float2(-INFINITY, 0.f);
      if (j < ns) v = __ldcg(reinterpret_cast<const float2*>(pml_a + ((row0 + g) * slots_a + s0 + j) * 2));
      mls[g][j] = v;
    }
    float pv[G][8];
    if (tid < D) {
#pragma unroll
      for (int g = 0; g < G; ++g)
#pragma unroll
        for (int j = 0; j < 8; ++j)
          pv[g][j] = j < ns ? __ldcg(po_a + ((row0 + g) * slots_a + s0 + j) * D + tid) : 0.f;
    }
    __syncthreads();
    if (tid < D) {
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float cm = M[g];
#pragma unroll
        for (int j = 0; j < 8; ++j) cm = fmaxf(cm, mls[g][j].x);
        if (cm != -INFINITY) {
          const float sc = exp2f(M[g] - cm);                    // 0 while nothing was seen
          ll[g] *= sc;
          oo[g] *= sc;
#pragma unroll
          for (int j = 0; j < 8; ++j) {                        // slots past ns: m = -inf, f = 0
            const float f = exp2f(mls[g][j].x - cm);
            ll[g] = fmaf(mls[g][j].y, f, ll[g]);
            oo[g] = fmaf(pv[g][j], f, oo[g]);
          }
          M[g] = cm;
        }
      }
    }
  }
  if (tid >= D) return;
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const int64_t row = row0 + g;
    const float r = ll[g] != 0.f ? oo[g] / ll[g] : 0.f;        // NaN l (a timed-out piece): NaN
    if constexpr (sizeof(OutT) == 4) out[row * D + tid] = r;
    else out[row * D + tid] = __float2bfloat16_rn(r);
  }
}

}  // namespace kvq

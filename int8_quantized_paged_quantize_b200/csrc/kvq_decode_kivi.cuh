// Paged GQA decode attention over the KIVI-style low-bit cache (2- or 4-bit
// codes, K per channel over 128-token groups, V per token), on the 5th
// generation tensor cores. A 128-token tile of a sequence is exactly one K
// group, so every tile has its own per-channel (s, z) for K and per-token
// (s, z) for V:
//   S[t][g] = sum_d q_gd (s_d c_td + z_d) = sum_d (q_gd s_d) c_td + sum_d q_gd z_d
//   O[g][d] = sum_t p_gt (s_t c_td + z_t) = sum_t (p_gt s_t) c_td + sum_t p_gt z_t
// The codes are the unsigned 8-bit MMA operands (kind::i8): the query of every
// tile is rebuilt with the tile's channel scales (three exact s8 parts, as for
// static INT8) and the weights p s_t are the three bytes of a 24-bit fixed
// point (as for INT8); the z terms are added in FP32. Included by
// kvq_kernels.cu after kvq_decode_mma.cuh (PieceWalk, tmem_load_cols).
//
// Pages arrive packed (b bits per code, 16 codes in 2b bytes) and are
// expanded in shared memory into the 8-bit operand layouts of the 8-bit
// formats (one shift and one mask per four output bytes). Rings: packed
// stages (producer -> expanding warps) and operand stages (-> MMA) are
// separate, so that more copies are in flight than operand stages fit.
//
// 8 warps per CTA:
//   warp 0      producer: lanes 0..7 copy one packed K and V page each of a
//               128-token tile (1-D bulk copies); every lane stores 16 bytes of
//               the tile's K and V (s, z) pairs into the packed stage.
//   warp 1      TMEM allocation; one thread issues the MMAs.
//   warps 2..5  softmax warps: thread r owns token r (S, P) and channel r (O);
//               at the end of a tile they expand the next tile's V pages
//               (whose stage the PV product two tiles back has released).
//   warps 6..7  converters: expand the K pages and rebuild the query operand
//               of every tile from its K channel scales (each warp half of the
//               heads); they run ahead of the softmax warps, so the rebuild is
//               off the softmax warps' per-tile chain.
// Every wait is bounded as in the 8-bit kernel; on expiry the CTA drains what
// it issued, writes NaN markers for its partials, frees TMEM and returns.
// The tokens after the last complete group are not in this cache: a BF16
// residual cache holds them and a second partial pass covers them.

#pragma once

namespace kvq {

template <int D, int G, int BITS>
struct KiviCfg {
  static constexpr int PAGE = kBlockSize * D;                 // operand page bytes (u8 codes)
  static constexpr int PPAGE = kBlockSize * D * BITS / 8;     // packed page bytes
  static constexpr int NST = 2;                               // operand stages
  static constexpr int NSP = BITS == 2 ? 3 : 2;               // packed stages
  static constexpr int META = kBlockSize * 2 * 2;             // (s, z) bytes per page
  static constexpr int QPARTS = 3, PPARTS = 3;
  static constexpr int NS = round_up16(QPARTS * G);
  static constexpr int NO = round_up16(PPARTS * G);
  static constexpr int NSL = (QPARTS * G + 7) / 8 * 8;
  static constexpr int NOL = (PPARTS * G + 7) / 8 * 8;
  static_assert(NS <= 32 && NO <= 32, "query group too large");
  static constexpr int S_MMAS = D / 32;
  static constexpr int PV_MMAS = 128 / 32;
  static constexpr uint32_t K_LBO = 128, K_SBO = 8 * D;
  static constexpr uint32_t V_LBO = 16 * D, V_SBO = 128;
  static constexpr uint32_t Q_SBO = 128, Q_LBO = (NS / 8) * 128;
  static constexpr uint32_t P_SBO = 128, P_LBO = (NO / 16) * 128;
  static constexpr int QBYTES = NS * D;
  static constexpr int PBYTES = NO * 128;
  static constexpr int COL_S = 0, COL_O = 64, TMEM_COLS = 128;
  // shared memory (offsets from a 128-byte aligned base)
  static constexpr int OFF_K = 0;                                   // [NST][8 pages]
  static constexpr int OFF_V = OFF_K + NST * 8 * PAGE;
  static constexpr int OFF_PK = OFF_V + NST * 8 * PAGE;             // [NSP][8 packed pages]
  static constexpr int OFF_PV = OFF_PK + NSP * 8 * PPAGE;
  static constexpr int OFF_PKM = OFF_PV + NSP * 8 * PPAGE;          // [NSP][8][META]
  static constexpr int OFF_PVM = OFF_PKM + NSP * 8 * META;
  static constexpr int OFF_Q = (OFF_PVM + NSP * 8 * META + 127) / 128 * 128;
  static constexpr int OFF_P = OFF_Q + QBYTES;                      // [2]
  static constexpr int OFF_BAR = OFF_P + 2 * PBYTES;
  static constexpr int NBAR = 2 * NSP + 4 * NST + 10 + 3 + 4;
  static constexpr int OFF_RED = (OFF_BAR + 8 * NBAR + 15) / 16 * 16;   // float [2][64]; prologue
  static constexpr int OFF_RED2 = OFF_RED + 2 * 4 * 16 * 4;        // float [2][4][8]
  static constexpr int OFF_QSC = OFF_RED2 + 2 * 4 * 8 * 4;         // float [4][8] scale, [4][8] sum(q z)
  static constexpr int OFF_PMASK = OFF_QSC + 64 * 4;               // uint32 [NSP] page masks
  static constexpr int OFF_MISC = (OFF_PMASK + 4 * NSP + 15) / 16 * 16;
  static constexpr int OFF_WALK = OFF_MISC + 32;
  static constexpr int SMEM = OFF_WALK + 160 + 128;
  static_assert(OFF_RED % 16 == 0 && OFF_BAR % 8 == 0 && OFF_MISC % 16 == 0, "smem alignment");
  static_assert(OFF_PK % 16 == 0 && OFF_PKM % 16 == 0, "bulk copy alignment");
};

// Expand the packed codes of one 128-token tile's 8 pages (K or V) into the
// 8-bit operand layout, by NT threads (t = 0 .. NT-1). 16 operand bytes (one
// 16-byte row of a core matrix) come from one packed 32-bit word (2-bit codes:
// bit pair k of packed byte j is operand byte 4k + j) or one 64-bit word
// (4-bit: the low and high nibbles of packed byte j of word i are operand
// bytes 8i + j and 8i + 4 + j). Consecutive threads take consecutive 16-byte
// rows, so neither the packed reads nor the operand writes of a warp meet a
// shared-memory bank twice; the packed words of a batch are all read before
// any operand row is written (the two may alias as far as the compiler
// knows), so a batch costs one shared-memory round trip.
template <class C, int BITS, int NT>
__device__ __forceinline__ void kivi_expand(const uint8_t* psrc, uint8_t* odst, int t) {
  uint4* dst = reinterpret_cast<uint4*>(odst);
  constexpr int PER = 8 * C::PAGE / 16 / NT;                // 16-byte rows per thread
  constexpr int BATCH = PER < 8 ? PER : 8;
  static_assert(PER * NT * 16 == 8 * C::PAGE && PER % BATCH == 0, "rows per thread");
#pragma unroll
  for (int b0 = 0; b0 < PER; b0 += BATCH) {
    if constexpr (BITS == 2) {
      uint32_t w[BATCH];
#pragma unroll
      for (int k = 0; k < BATCH; ++k) w[k] = reinterpret_cast<const uint32_t*>(psrc)[t + NT * (b0 + k)];
#pragma unroll
      for (int k = 0; k < BATCH; ++k)
        dst[t + NT * (b0 + k)] = make_uint4(w[k] & 0x03030303u, (w[k] >> 2) & 0x03030303u,
                                            (w[k] >> 4) & 0x03030303u, (w[k] >> 6) & 0x03030303u);
    } else {
      uint2 w[BATCH];
#pragma unroll
      for (int k = 0; k < BATCH; ++k) w[k] = reinterpret_cast<const uint2*>(psrc)[t + NT * (b0 + k)];
#pragma unroll
      for (int k = 0; k < BATCH; ++k)
        dst[t + NT * (b0 + k)] = make_uint4(w[k].x & 0x0F0F0F0Fu, (w[k].x >> 4) & 0x0F0F0F0Fu,
                                            w[k].y & 0x0F0F0F0Fu, (w[k].y >> 4) & 0x0F0F0F0Fu);
    }
  }
}

// The BF16 query rows of heads gs[0 .. HN) (-1: none) of one (sequence, KV
// head) group starting at `rows`, as floats; lane owns the D/32 consecutive
// channels lane * D/32 ...
template <int D, int HN>
__device__ __forceinline__ void kivi_load_query(float (&qr)[HN][D / 32], const int (&gs)[HN],
                                                const __nv_bfloat16* rows, bool none, int lane) {
  constexpr int CPL = D / 32;
  const int d0 = lane * CPL;
#pragma unroll
  for (int hh = 0; hh < HN; ++hh) {
    uint32_t w[CPL / 2];
#pragma unroll
    for (int i = 0; i < CPL / 2; ++i) w[i] = 0u;
    if (gs[hh] >= 0 && !none) {
      const __nv_bfloat16* src = rows + int64_t(gs[hh]) * D + d0;
      if constexpr (CPL == 4) {
        const uint2 u = *reinterpret_cast<const uint2*>(src);
        w[0] = u.x; w[1] = u.y;
      } else {
        w[0] = *reinterpret_cast<const uint32_t*>(src);
      }
    }
#pragma unroll
    for (int i = 0; i < CPL / 2; ++i) {
      qr[hh][2 * i] = __uint_as_float(w[i] << 16);
      qr[hh][2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
}

// The query operand rows of heads gs[0 .. HN) for one tile: x = q s_d (the
// tile's K channel scales, from the (s, z) pairs `kpairs` of its packed stage)
// in three exact s8 parts after a power-of-two scaling of the head, written
// into `qop` (rows j * G + g); qsc_slot[g] = qk_scale * 2^-e and
// qzs_slot[g] = qk_scale * sum_d q z_d. The lane's consecutive channels make
// one word (or half word) per part. Warp-collective.
template <class C, int D, int G, int HN>
__device__ __forceinline__ void kivi_build_query(const float (&qc)[HN][D / 32], const int (&gs)[HN],
                                                 const uint8_t* kpairs, uint8_t* qop, float* qsc_slot,
                                                 float* qzs_slot, float qk_scale, int lane) {
  using namespace tc;
  constexpr int CPL = D / 32;
  const int d0 = lane * CPL;
  // the tile's K (s, z) pairs, in the packed stage the producer filled;
  // channel d: page d / (D/8), entry d % (D/8); the lane's channels are
  // consecutive entries of one page
  const __nv_bfloat162* kmp = reinterpret_cast<const __nv_bfloat162*>(kpairs) +
                              (d0 / (D / 8)) * kBlockSize + d0 % (D / 8);
  float sd[CPL], zd[CPL];
  {
    __nv_bfloat162 pr[CPL];
    if constexpr (CPL == 4) {
      const uint4 u = *reinterpret_cast<const uint4*>(kmp);
      *reinterpret_cast<uint4*>(pr) = u;
    } else {
      const uint2 u = *reinterpret_cast<const uint2*>(kmp);
      *reinterpret_cast<uint2*>(pr) = u;
    }
#pragma unroll
    for (int i = 0; i < CPL; ++i) { sd[i] = __low2float(pr[i]); zd[i] = __high2float(pr[i]); }
  }
  // all of the warp's heads at once, so that their reductions overlap
  float x[HN][CPL], zsum[HN];
  uint32_t amax[HN];
#pragma unroll
  for (int hh = 0; hh < HN; ++hh) {
    float zs = 0.f, am = 0.f;
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
      x[hh][i] = qc[hh][i] * sd[i];
      zs = fmaf(qc[hh][i], zd[i], zs);
      am = fmaxf(am, fabsf(x[hh][i]));
    }
    zsum[hh] = zs;
    amax[hh] = __float_as_uint(am);
  }
  // the head's largest |x|: one integer reduction on the float bits (x >= 0)
#pragma unroll
  for (int hh = 0; hh < HN; ++hh) amax[hh] = __reduce_max_sync(0xffffffffu, amax[hh]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1)
#pragma unroll
    for (int hh = 0; hh < HN; ++hh) zsum[hh] += __shfl_xor_sync(0xffffffffu, zsum[hh], o);
#pragma unroll
  for (int hh = 0; hh < HN; ++hh) {
    const int g = gs[hh];
    // e = 5 - floor(log2 amax) from the exponent field (zero and subnormal
    // maxima clamp to 120, infinities to -120)
    int e = 0;
    if (amax[hh] != 0u) e = 5 - (int(amax[hh] >> 23) - 127);
    e = max(-120, min(120, e));
    const float up = __int_as_float((127 + e) << 23);
    const float down = __int_as_float((127 - e) << 23);
    // the three parts by rounding additions (1.5 * 2^23 + v holds rint(v)
    // in its low bits for |v| < 2^22): t_j's low byte is part j's code
    constexpr float kMg = 12582912.0f;
    uint32_t tb[3][CPL];
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
      const float xs = x[hh][i] * up;
      const float t0 = __fadd_rn(xs, kMg), x0 = __fsub_rn(t0, kMg);
      const float r0 = (xs - x0) * 128.f;
      const float t1 = __fadd_rn(r0, kMg), x1 = __fsub_rn(t1, kMg);
      const float t2 = __fadd_rn((r0 - x1) * 128.f, kMg);
      tb[0][i] = __float_as_uint(t0);
      tb[1][i] = __float_as_uint(t1);
      tb[2][i] = __float_as_uint(t2);
    }
    uint32_t part[3];
#pragma unroll
    for (int j = 0; j < 3; ++j) {
      if constexpr (CPL == 4)
        part[j] = __byte_perm(__byte_perm(tb[j][0], tb[j][1], 0x0040), __byte_perm(tb[j][2], tb[j][3], 0x0040), 0x5410);
      else
        part[j] = __byte_perm(tb[j][0], tb[j][1], 0x0040) & 0xFFFFu;
    }
    if (g >= 0) {
#pragma unroll
      for (int j = 0; j < 3; ++j) {
        const int n = j * G + g;                         // operand row of this part
        uint8_t* at = qop + (n >> 3) * C::Q_SBO + (n & 7) * 16 + (d0 >> 4) * C::Q_LBO + (d0 & 15);
        if constexpr (CPL == 4) *reinterpret_cast<uint32_t*>(at) = part[j];
        else *reinterpret_cast<uint16_t*>(at) = uint16_t(part[j]);
      }
      if (lane == 0) {
        qsc_slot[g] = qk_scale * down;
        qzs_slot[g] = qk_scale * zsum[hh];
      }
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
}

template <int D, int G, int BITS>
__global__ void __launch_bounds__(256, 2) decode_kivi_kernel(
    const __nv_bfloat16* __restrict__ q, const uint8_t* __restrict__ kc,
    const uint8_t* __restrict__ vc, const __nv_bfloat16* __restrict__ km,
    const __nv_bfloat16* __restrict__ vm, const int32_t* __restrict__ tables,
    const int32_t* __restrict__ ctx_lens, int B, int Hk, int NB, int W, int max_ctx,
    int unit_tiles, int slots, float qk_scale, long long wait_limit, float* __restrict__ part_o,
    float* __restrict__ part_ml, int32_t* __restrict__ part_cnt) {
  using C = KiviCfg<D, G, BITS>;
  using namespace tc;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((128 - (smem_u32(smem_raw) & 127)) & 127);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int Hq = Hk * G;
  constexpr int NWARPS = 8;

  // ------------------------------------------------------------ the share
  long long* red64 = reinterpret_cast<long long*>(smem + C::OFF_RED);
  long long* miscll = reinterpret_cast<long long*>(smem + C::OFF_MISC + 16);
  int* misci = reinterpret_cast<int*>(smem + C::OFF_MISC + 8);
  {
    long long tsum = 0;
    for (int bb = threadIdx.x; bb < B; bb += blockDim.x) {
      const int c = ctx_lens[bb];
      if (c < 0 || c > max_ctx || int64_t(c) > int64_t(W) * kBlockSize || (c & 127) != 0) {
        if (blockIdx.x == 0) flag_error(KVQ_DEVERR_CONTEXT);
      }
      const int cg = mma_seq_ctx(ctx_lens, bb, max_ctx, W) & ~127;   // whole groups only
      if (cg > 0) tsum += cg / 128 + kPieceCost;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) tsum += __shfl_xor_sync(0xffffffffu, tsum, o);
    if (lane == 0) red64[warp] = tsum;
  }
  __syncthreads();
  long long T = 0;
#pragma unroll
  for (int w = 0; w < NWARPS; ++w) T += red64[w];
  T *= Hk;
  const long long N = ll_min(gridDim.x, ll_max(1, T / max(1, unit_tiles)));
  if (T == 0 || blockIdx.x >= N) return;
  const long long start = (int64_t(blockIdx.x) * T) / N;
  const long long end = (int64_t(blockIdx.x + 1) * T) / N;
  // a length that is not a whole number of groups is cut to its whole groups
  // (and flagged above); the walk below cuts it the same way
  auto seq_ctx = [&](int bb) -> int { return mma_seq_ctx(ctx_lens, bb, max_ctx, W) & ~127; };
  {
    if (threadIdx.x == 0) misci[0] = -1;
    __syncthreads();
    long long run = 0;
    for (int base = 0; base < B; base += blockDim.x) {
      const int bb = base + threadIdx.x;
      int tb = bb < B ? seq_ctx(bb) / 128 : 0;
      if (tb > 0) tb += kPieceCost;
      long long incl = tb;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const long long y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      __syncthreads();
      if (lane == 31) red64[warp] = incl;
      __syncthreads();
      long long before = 0, total = 0;
#pragma unroll
      for (int w = 0; w < NWARPS; ++w) {
        before += (w < warp) ? red64[w] : 0;
        total += red64[w];
      }
      const long long lo_t = run + before + incl - tb;
      if (bb < B && tb > 0 && int64_t(Hk) * lo_t <= start && start < int64_t(Hk) * (lo_t + tb)) {
        misci[0] = bb;
        miscll[0] = lo_t;
      }
      run += total;
      __syncthreads();
      if (misci[0] >= 0) break;
    }
  }
  const int b0 = misci[0];
  const long long P0 = miscll[0];
  auto cta_of = [&](long long x) -> long long { return ((x + 1) * N - 1) / T; };

  uint8_t* kring = smem + C::OFF_K;
  uint8_t* vring = smem + C::OFF_V;
  uint8_t* pkring = smem + C::OFF_PK;
  uint8_t* pvring = smem + C::OFF_PV;
  uint8_t* pkmeta = smem + C::OFF_PKM;
  uint8_t* pvmeta = smem + C::OFF_PVM;
  uint8_t* qop = smem + C::OFF_Q;
  uint8_t* pop = smem + C::OFF_P;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* pfull = bars;                      // [NSP] producer -> converters (K and V)
  uint64_t* pfree = pfull + C::NSP;            // [NSP] converters -> producer
  uint64_t* kready = pfree + C::NSP;           // [NST] converters -> MMA, softmax
  uint64_t* kempty = kready + C::NST;          // [NST] softmax -> converters
  uint64_t* vready = kempty + C::NST;          // [NST]
  uint64_t* vempty = vready + C::NST;          // [NST] MMA (PV done) -> converters
  uint64_t* sfull = vempty + C::NST;           // [2]
  uint64_t* sfree = sfull + 2;
  uint64_t* pready = sfree + 2;
  uint64_t* ofull = pready + 2;
  uint64_t* ofree = ofull + 2;
  uint64_t* qready = ofree + 2;
  uint64_t* qfree = qready + 1;
  uint64_t* drain = qfree + 1;
  uint64_t* qinfo = drain + 1;                 // [4] converters -> softmax (qsc, qzs)
  float* red = reinterpret_cast<float*>(smem + C::OFF_RED);
  float* red2 = reinterpret_cast<float*>(smem + C::OFF_RED2);
  float* qsc = reinterpret_cast<float*>(smem + C::OFF_QSC);      // [4][8]
  float* qzs = qsc + 32;                                           // [4][8]
  volatile uint32_t* pmask_p = reinterpret_cast<volatile uint32_t*>(smem + C::OFF_PMASK);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  // ------------------------------------------------------------ set-up
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NSP; ++s) {
      mbar_init(pfull + s, 1);
      mbar_init(pfree + s, 64 + 128);             // converters (K) and softmax warps (V)
    }
    for (int s = 0; s < C::NST; ++s) {
      mbar_init(kready + s, 64);
      mbar_init(kempty + s, 128);
      mbar_init(vready + s, 128);
      mbar_init(vempty + s, 1);
    }
    for (int j = 0; j < 2; ++j) {
      mbar_init(sfull + j, 1);
      mbar_init(sfree + j, 128);
      mbar_init(pready + j, 128);
      mbar_init(ofull + j, 1);
      mbar_init(ofree + j, 128);
    }
    mbar_init(qready, 64);
    mbar_init(qfree, 1);
    for (int j = 0; j < 4; ++j) mbar_init(qinfo + j, 64);
    mbar_init(drain, 1);
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp >= 2 && warp < 6) {
    const int ct = threadIdx.x - 64;
    for (int i = ct * 16; i < C::QBYTES + 2 * C::PBYTES; i += 128 * 16)
      *reinterpret_cast<uint4*>(qop + i) = make_uint4(0, 0, 0, 0);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto walk_next = [&](PieceWalk& pw) {
    // step over runs of sequences whose length is not whole groups
    pw.next(Hk, ctx_lens, B, max_ctx, W);
  };
  PieceWalk walk;
  walk.init(b0, P0, start, end, Hk, ctx_lens, B, max_ctx, W, ~127);

  if (warp == 0) {
    // ---------------------------------------------------------- producer
    const uint64_t pol = l2_evict_first_policy();
    const int p8 = lane & 7;
    auto load_id = [&](const PieceWalk& pw, int tile) -> int {
      if (lane >= 8 || pw.done) return -2;
      const int tok0 = tile * 128;
      const int t1 = min(pw.hi * 128, pw.ctx);
      const int npg = min(8, (t1 - tok0 + kBlockSize - 1) / kBlockSize);
      return p8 < npg ? tables[int64_t(pw.b) * W + tok0 / kBlockSize + p8] : -2;
    };
    auto step = [&](PieceWalk& pw, int& tile) {
      if (pw.done) return;
      if (++tile >= pw.hi) {
        walk_next(pw);
        tile = pw.lo;
      }
    };
    // lane l: 16-byte chunk l % 4 of page l / 4 ... 8 pages x 64 bytes = 32 chunks
    const int sp_pg = lane >> 2, sp_c = lane & 3;
    auto load_meta = [&](int ids, int h, uint4& kv, uint4& vv) {
      kv = vv = make_uint4(0, 0, 0, 0);
      const int sblk = __shfl_sync(0xffffffffu, ids, sp_pg);
      if (sblk >= 0 && sblk < NB) {
        const int64_t off = (int64_t(sblk) * Hk + h) * C::META + sp_c * 16;
        kv = __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(km) + off));
        vv = __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(vm) + off));
      }
    };
    PieceWalk c0 = walk, c1 = walk, c2 = walk;
    int i0 = walk.lo, i1 = walk.lo, i2 = walk.lo;
    step(c1, i1);
    step(c2, i2);
    step(c2, i2);
    int id0 = load_id(c0, i0), id1 = load_id(c1, i1);
    uint4 kmv, vmv;
    load_meta(id0, c0.h, kmv, vmv);
    bool iss[C::NSP];
    uint32_t par[C::NSP];
#pragma unroll
    for (int s = 0; s < C::NSP; ++s) { iss[s] = false; par[s] = 0; }
    for (int gt = 0; !c0.done; ++gt) {
      const int s = gt % C::NSP;
      const uint32_t ph = (gt / C::NSP) & 1;
      const int h = c0.h;
      const int id = id0;
      const int id2 = load_id(c2, i2);
      uint4 kmn, vmn;
      load_meta(c1.done ? -2 : id1, c1.h, kmn, vmn);
      if (lane < 8 && id != -2 && (id < 0 || id >= NB)) flag_error(KVQ_DEVERR_BLOCK);
      const bool valid = lane < 8 && id >= 0 && id < NB;
      const uint32_t mask = __ballot_sync(0xffffffffu, valid) & 0xFFu;
      const int blk = __shfl_sync(0xffffffffu, id, p8);
      const bool mine = ((mask >> p8) & 1u) != 0u;
      const int64_t page = int64_t(blk) * Hk + h;
      const uint32_t bytes = 2u * uint32_t(__popc(mask)) * uint32_t(C::PPAGE);
      bool ok = true;
      if (lane == 0) {
        ok = mbar_wait(pfree + s, ph ^ 1, abort_flag, wait_limit);
        if (ok) mbar_expect_tx(pfull + s, bytes);
      }
      if (!__shfl_sync(0xffffffffu, int(ok), 0)) break;
      if (lane < 8 && mine) {
        bulk_g2s(pkring + (s * 8 + p8) * C::PPAGE, kc + page * C::PPAGE, C::PPAGE, pfull + s, pol);
        bulk_g2s(pvring + (s * 8 + p8) * C::PPAGE, vc + page * C::PPAGE, C::PPAGE, pfull + s, pol);
      }
      iss[s] = true;
      par[s] = ph;
      *reinterpret_cast<uint4*>(pkmeta + (s * 8 + sp_pg) * C::META + sp_c * 16) = kmv;
      *reinterpret_cast<uint4*>(pvmeta + (s * 8 + sp_pg) * C::META + sp_c * 16) = vmv;
      __syncwarp();
      if (lane == 0) {
        pmask_p[s] = mask;
        mbar_arrive(pfull + s);
      }
      c0 = c1; i0 = i1; id0 = id1; kmv = kmn; vmv = vmn;
      c1 = c2; i1 = i2; id1 = id2;
      step(c2, i2);
    }
    if (lane == 0 && *abort_flag) {
      volatile int no_abort = 0;
      for (int s = 0; s < C::NSP; ++s)
        if (iss[s]) mbar_wait(pfull + s, par[s], &no_abort, kMmaWaitLimitCycles);
    }
  } else if (warp >= 6) {
    // ---------------------------------------------------------- converters
    const int ct = threadIdx.x - 192;                       // 0..63
    const int cw = warp - 6;
    // the query operand of every tile: heads cw, cw + 2, ... (the converters
    // run several tiles ahead of the softmax warps, so the rebuild is off the
    // softmax warps' per-tile chain)
    constexpr int HPC = (G + 1) / 2;
    constexpr int CPL = D / 32;
    int gsc[HPC];
#pragma unroll
    for (int hh = 0; hh < HPC; ++hh) gsc[hh] = cw + 2 * hh < G ? cw + 2 * hh : -1;
    auto rows_of = [&](const PieceWalk& pw) { return q + (int64_t(pw.b) * Hq + int64_t(pw.h) * G) * D; };
    bool ok = true;
    int gt = 0;
    float qcur[HPC][CPL], qnext[HPC][CPL];
    kivi_load_query<D, HPC>(qcur, gsc, walk.done ? q : rows_of(walk), walk.done, lane);
    for (PieceWalk pw = walk; !pw.done;) {
      PieceWalk nx = pw;
      walk_next(nx);
      kivi_load_query<D, HPC>(qnext, gsc, nx.done ? q : rows_of(nx), nx.done, lane);   // a piece ahead
      for (int i = pw.lo; i < pw.hi; ++i, ++gt) {
        const int sp = gt % C::NSP, su = gt % C::NST;
        if (ok) ok = mbar_wait(pfull + sp, (gt / C::NSP) & 1, abort_flag, wait_limit);
        // K operand stage free: the S product of its last tile has been read
        if (ok) ok = mbar_wait(kempty + su, ((gt / C::NST) & 1) ^ 1, abort_flag, wait_limit);
        if (ok) {
          kivi_expand<C, BITS, 64>(pkring + sp * 8 * C::PPAGE, kring + su * 8 * C::PAGE, ct);
          fence_proxy_async_smem();
        }
        mbar_arrive(kready + su);
        // this warp's heads of the tile's query operand (the previous tile's S
        // product has read the operand)
        if (ok && gt > 0) ok = mbar_wait(qfree, (gt - 1) & 1, abort_flag, wait_limit);
        ok = __all_sync(0xffffffffu, ok);                   // the build is warp-collective
        if (ok)
          kivi_build_query<C, D, G, HPC>(qcur, gsc, pkmeta + sp * 8 * C::META, qop, qsc + (gt & 3) * 8,
                                         qzs + (gt & 3) * 8, qk_scale, lane);
        mbar_arrive(qready);
        mbar_arrive(qinfo + (gt & 3));
        mbar_arrive(pfree + sp);                          // the softmax warps expand V
      }
#pragma unroll
      for (int hh = 0; hh < HPC; ++hh)
#pragma unroll
        for (int i = 0; i < CPL; ++i) qcur[hh][i] = qnext[hh][i];
      pw = nx;
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      // A: u8 codes; B: s8 query parts (S), u8 weight parts (PV); s32 sums
      constexpr uint32_t id_s = idesc_m128(2u, 0u, 1u, false, C::NS);
      constexpr uint32_t id_pv = idesc_m128(2u, 0u, 0u, true, C::NO);
      const uint32_t kbase = smem_u32(kring), vbase = smem_u32(vring);
      const uint32_t qaddr = smem_u32(qop), paddr = smem_u32(pop);
      bool ok = true;
      int gt = 0;
      auto issue_pv = [&](int j) -> bool {
        const int s = j % C::NST;
        if (!mbar_wait(pready + (j & 1), (j >> 1) & 1, abort_flag, wait_limit)) return false;
        if (!mbar_wait(ofree + (j & 1), ((j >> 1) & 1) ^ 1, abort_flag, wait_limit)) return false;
        if (!mbar_wait(vready + s, (j / C::NST) & 1, abort_flag, wait_limit)) return false;
        tc_fence_after();
        const uint32_t a0 = vbase + s * 8 * C::PAGE;
        const uint32_t b0 = paddr + (j & 1) * C::PBYTES;
#pragma unroll
        for (int kk = 0; kk < C::PV_MMAS; ++kk)
          mma_ss<2>(tmem + C::COL_O + (j & 1) * 32, sdesc_plain(a0 + kk * 2 * C::V_LBO, C::V_LBO, C::V_SBO),
                    sdesc_plain(b0 + kk * 4 * C::P_LBO, C::P_LBO, C::P_SBO), id_pv, kk > 0);
        mma_commit(ofull + (j & 1));
        mma_commit(vempty + s);
        return true;
      };
      for (; ok && !walk.done; walk_next(walk)) {
        for (int i = walk.lo; ok && i < walk.hi; ++i, ++gt) {
          const int s = gt % C::NST;
          // the query of tile gt (rebuilt for every tile), its K stage, an S buffer
          ok = mbar_wait(qready, gt & 1, abort_flag, wait_limit) &&
               mbar_wait(kready + s, (gt / C::NST) & 1, abort_flag, wait_limit) &&
               mbar_wait(sfree + (gt & 1), ((gt >> 1) & 1) ^ 1, abort_flag, wait_limit);
          if (!ok) break;
          tc_fence_after();
          const uint32_t a0 = kbase + s * 8 * C::PAGE;
#pragma unroll
          for (int kk = 0; kk < C::S_MMAS; ++kk)
            mma_ss<2>(tmem + C::COL_S + (gt & 1) * 32, sdesc_plain(a0 + kk * 2 * C::K_LBO, C::K_LBO, C::K_SBO),
                      sdesc_plain(qaddr + kk * 2 * C::Q_LBO, C::Q_LBO, C::Q_SBO), id_s, kk > 0);
          mma_commit(sfull + (gt & 1));
          mma_commit(qfree);                               // the query may be rebuilt
          if (gt >= 1) ok = issue_pv(gt - 1);
        }
      }
      if (ok && gt >= 1) issue_pv(gt - 1);
      volatile int no_abort = 0;
      mma_commit(drain);
      mbar_wait(drain, 0, &no_abort, kMmaWaitLimitCycles);
    }
  } else {
    // ---------------------------------------------------------- softmax warps
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_base = uint32_t(quarter * 32) << 16;
    bool ok = true;
    const uint32_t prow = (r >> 3) * C::P_LBO + (r & 7) * 16;
    PieceWalk* wk = reinterpret_cast<PieceWalk*>(smem + C::OFF_WALK);
    int* pinfo = reinterpret_cast<int*>(smem + C::OFF_WALK + 2 * sizeof(PieceWalk));
    auto publish = [&](int idx, const PieceWalk& pw) {
      wk[idx] = pw;
      if (!pw.done) {
        pinfo[idx * 2] = int(int64_t(blockIdx.x) - cta_of(pw.first_tile(Hk)));
        pinfo[idx * 2 + 1] = pw.hi == pw.nt;
      }
    };
    if (r == 0) {
      publish(0, walk);
      PieceWalk n = walk;
      walk_next(n);
      publish(1, n);
    }
    named_bar_sync(1, 128);

    // the V codes of a tile, expanded by these warps one tile ahead (at the end
    // of the previous tile, whose PV product has been issued by then), with
    // the tile's page mask and this token's V (s, z) kept in registers
    uint32_t vmask_n = 0u;
    float sv_n = 0.f, zv_n = 0.f;
    auto stage_v = [&](int gv) {
      const int sp = gv % C::NSP, su = gv % C::NST;
      if (ok) ok = mbar_wait(pfull + sp, (gv / C::NSP) & 1, abort_flag, wait_limit);
      // V operand stage free: the PV product of its last tile has completed
      if (ok) ok = mbar_wait(vempty + su, ((gv / C::NST) & 1) ^ 1, abort_flag, wait_limit);
      if (ok) {
        kivi_expand<C, BITS, 128>(pvring + sp * 8 * C::PPAGE, vring + su * 8 * C::PAGE, r);
        vmask_n = pmask_p[sp];
        const __nv_bfloat162 vmp =
            reinterpret_cast<const __nv_bfloat162*>(pvmeta + (sp * 8 + (r >> 4)) * C::META)[r & 15];
        sv_n = __low2float(vmp);
        zv_n = __high2float(vmp);
        fence_proxy_async_smem();
      }
      mbar_arrive(vready + su);
      mbar_arrive(pfree + sp);
    };
    if (!wk[0].done) stage_v(0);

    int gt = 0;
    for (int pc = 0;; ++pc) {
      const PieceWalk* cur = wk + (pc & 1);
      const PieceWalk* nxt = wk + ((pc + 1) & 1);
      if (cur->done) break;
      const int pb = cur->b, ph_ = cur->h, lo = cur->lo, hi = cur->hi;
      const int t1 = min(hi * 128, cur->ctx);
      const int slot = pinfo[(pc & 1) * 2], last = pinfo[(pc & 1) * 2 + 1];
      const bool more = !nxt->done;
      named_bar_sync(1, 128);
      if (r == 0) {
        PieceWalk n = *nxt;
        if (!n.done) walk_next(n);
        publish(pc & 1, n);
      }
      float m[G], l[G], corr[G], o[G], alpha[G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        m[g] = -INFINITY; l[g] = 0.f; corr[g] = 0.f; o[g] = 0.f; alpha[g] = 1.f;
      }
      float einv_pend = 1.f;

      auto accum_o = [&](int j) {
        if (ok) ok = mbar_wait(ofull + (j & 1), (j >> 1) & 1, abort_flag, wait_limit);
        tc_fence_after();
        uint32_t ov[C::NOL];
        if (ok) {
          tmem_load_cols<C::NOL>(tmem + lane_base + C::COL_O + (j & 1) * 32, ov);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int e = 0; e < C::NOL; ++e) ov[e] = 0u;
        }
        tc_fence_before();
        mbar_arrive(ofree + (j & 1));
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float v = float(int(ov[g])) + float(int(ov[G + g])) * (1.f / 256.f) +
                          float(int(ov[2 * G + g])) * (1.f / 65536.f);
          o[g] += v * (einv_pend * alpha[g]);
        }
      };

      for (int i = lo; i < hi; ++i, ++gt) {
        const int su = gt % C::NST;
        if (ok) ok = mbar_wait(sfull + (gt & 1), (gt >> 1) & 1, abort_flag, wait_limit);
        tc_fence_after();
        uint32_t sw[C::NSL];
        if (ok) {
          tmem_load_cols<C::NSL>(tmem + lane_base + C::COL_S + (gt & 1) * 32, sw);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int e = 0; e < C::NSL; ++e) sw[e] = 0u;
        }
        tc_fence_before();
        mbar_arrive(sfree + (gt & 1));
        // the K stage of this tile is free (its S product has been read)
        mbar_arrive(kempty + su);
        // the tile's per-head query factors, written with its query operand
        if (ok) ok = mbar_wait(qinfo + (gt & 3), (gt >> 2) & 1, abort_flag, wait_limit);
        float qs[G], qz[G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
          qs[g] = qsc[(gt & 3) * 8 + g];
          qz[g] = qzs[(gt & 3) * 8 + g];
        }

        // ---- this token's V (s, z), taken when the tile's V was expanded
        const uint32_t mask = ok ? vmask_n : 0u;
        const int tile0 = i * 128;
        const bool valid = ok && ((mask >> (r >> 4)) & 1u) && (tile0 + r < t1);
        const float sv = valid ? sv_n : 0.f, zv = valid ? zv_n : 0.f;
        float x[G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float sc = float(int(sw[g])) + float(int(sw[G + g])) * (1.f / 128.f) +
                           float(int(sw[2 * G + g])) * (1.f / 16384.f);
          x[g] = valid ? fmaf(sc, qs[g], qz[g]) : -INFINITY;
        }
        float* rb = red + (gt & 1) * 64;
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float tm = warp_max_f32(x[g]);
          if (lane == 0) rb[g * 4 + quarter] = tm;
        }
        {
          const float svm = warp_max_f32(sv);
          if (lane == 0) rb[8 * 4 + quarter] = svm;
        }
        named_bar_sync(1, 128);
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float4 t4 = *reinterpret_cast<const float4*>(rb + g * 4);
          const float tmax = fmaxf(fmaxf(t4.x, t4.y), fmaxf(t4.z, t4.w));
          const float mn = fmaxf(m[g], tmax);
          // 2^(m - mn) when the maximum moves, 1 while it stays (or while no
          // token has been seen): selects rather than branches, so that the
          // heads' exponentials overlap
          const float a = exp2f(m[g] - mn);
          alpha[g] = (mn == m[g] || mn == -INFINITY) ? 1.f : a;
          m[g] = mn;
          o[g] *= alpha[g];
        }
        const float4 s4 = *reinterpret_cast<const float4*>(rb + 8 * 4);
        const float svmax = fmaxf(fmaxf(s4.x, s4.y), fmaxf(s4.z, s4.w));
        int ex = 0;
        if (svmax > 0.f) ex = max(-120, min(120, 7 - (int(__float_as_uint(svmax) >> 23) - 127)));
        const float escale = __int_as_float((127 + ex) << 23);
        const float einv = __int_as_float((127 - ex) << 23);

        // ---- weights: Y = rint(p s_v 2^ex 2^16) < 2^24, its three bytes; the
        // z_v term sum_t p z_v in FP32
        uint8_t* pbuf = pop + (gt & 1) * C::PBYTES + prow;
        uint32_t yv[G];
        const float ysc = sv * escale * 65536.f;
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float e2 = exp2f(x[g] - m[g]);
          const float pr = x[g] != -INFINITY ? e2 : 0.f;
          l[g] = l[g] * alpha[g] + pr;
          yv[g] = __float2uint_rn(pr * ysc);
          corr[g] = corr[g] * alpha[g] + pr * zv;
        }
        uint32_t words[C::NO / 4];
#pragma unroll
        for (int e = 0; e < C::NO / 4; ++e) words[e] = 0u;
#pragma unroll
        for (int jj = 0; jj < 3; ++jj) {
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const int n = jj * G + g;
            words[n >> 2] |= ((yv[g] >> (16 - 8 * jj)) & 0xFFu) << (8 * (n & 3));
          }
        }
#pragma unroll
        for (int c16 = 0; c16 < C::NO / 16; ++c16)
          *reinterpret_cast<uint4*>(pbuf + c16 * C::P_SBO) =
              make_uint4(words[4 * c16], words[4 * c16 + 1], words[4 * c16 + 2], words[4 * c16 + 3]);
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(pready + (gt & 1));
        if (i > lo) accum_o(gt - 1);
        einv_pend = einv;
        // the next tile's V (it may open the next piece)
        if (i + 1 < hi || more) stage_v(gt + 1);
      }
#pragma unroll
      for (int g = 0; g < G; ++g) alpha[g] = 1.f;
      accum_o(gt - 1);

      // ---- piece partial
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float ls = warp_sum(l[g]);
        const float cs = warp_sum(corr[g]);
        if (lane == 0) {
          red2[quarter * 8 + g] = ls;
          red2[32 + quarter * 8 + g] = cs;
        }
      }
      named_bar_sync(1, 128);
      const bool good = ok && !*abort_flag;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float L = red2[g] + red2[8 + g] + red2[16 + g] + red2[24 + g];
        const float Cz = red2[32 + g] + red2[40 + g] + red2[48 + g] + red2[56 + g];
        const int64_t row = (int64_t(pb) * Hq + ph_ * G + g) * slots + slot;
        if (r < D) part_o[row * D + r] = good ? o[g] + Cz : __int_as_float(0x7fc00000);
        if (r == 0) {
          part_ml[row * 2] = good ? m[g] : INFINITY;
          part_ml[row * 2 + 1] = good ? L : __int_as_float(0x7fc00000);
        }
      }
      if (r == 0 && last) part_cnt[pb * Hk + ph_] = slot + 1;
      named_bar_sync(1, 128);                              // red2 is rewritten next piece
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
  if (threadIdx.x == 0 && *abort_flag) flag_error(KVQ_DEVERR_TIMEOUT);
}

}  // namespace kvq

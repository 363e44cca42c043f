// Chunked-prefill attention over the paged quantized cache with the query rows
// as the M dimension of the 5th-generation tensor-core products (the decode
// kernel puts the cache tokens there and fits at most 8 query rows per
// product). One CTA takes one block of 128 query rows of a (sequence, KV
// head) — the chunk's positions of the head's G query heads — over its share
// of the head's 128-token tiles, as a flash-attention loop:
//   S[128 rows x 64 tokens] = Q[128 x D] . K[64 x D]^T        (Q in shared
//                              memory, K codes expanded to f16 / bf16)
//   softmax in FP32 registers, one row per thread, over the tile's tokens,
//     with the per-token K scale (and zero point) applied to the columns
//   O[128 x D] += P'[128 x 64] . V[64 x D]                     (P' in tensor
//                              memory, V codes expanded to f16)
// where P' = p * v_scale of the token, kept to 22 bits as two f16 parts that
// share the FP32 accumulator (bf16 parts and the bf16 V pages as stored, for
// a BF16 cache). The cache codes are exact in f16 (E4M3, E5M2 and int8 values
// all are), the query is exact in bf16 and in f16 after a per-row
// power-of-two scaling, and the products accumulate in FP32, so the scores are
// those of the dequantized cache up to FP32 rounding. The online softmax keeps
// a lazily moved reference (it moves when the largest possible weight of a
// half tile, the score's exponential times the half's largest V scale, would
// exceed 2^8 relative to it), so P' stays within f16 range.
// Static INT8 scales vary along the contraction: the query is multiplied by
// the K scale of each channel and kept as two f16 parts; the V scale of each
// channel multiplies the finished row. Included by kvq_kernels.cu after
// kvq_decode_mma.cuh (PieceWalk, mma_seq_ctx, the tc wrappers).
//
// Work split: the work list is every (sequence, KV head, 128-token tile), as
// in the decode kernel; the nrb CTAs of a group (one per row block) walk the
// same share of it in step, so a page one of them copies from HBM is in L2
// for the others. Each piece ends in an online-softmax partial per row, and
// the merge kernel combines a row's partials (one count per row).
//
// 14 warps per CTA:
//   warp 0      producer: lanes 0..7 copy one K and one V page each of a tile
//               (1-D bulk copies) into a ring of raw stages and store the
//               pages' scales beside them.
//   warp 1      allocates TMEM; one thread issues the MMAs.
//   warps 2..9  softmax warps, two per TMEM lane quarter: thread r of a warp
//               owns query row r (TMEM lane r) for one half of a half tile's
//               columns (and of O's); the two exchange their row maxima and
//               sums through shared memory. They also build the query operand.
//   warps 10..13 converters: expand each half tile's K and V codes to f16 in a
//               converted stage, with V rows of tokens past the
//               sequence end or on invalid pages zeroed, and turn the
//               per-token scales into FP32 column factors. For a BF16 cache
//               they only zero those V rows in the raw stage.
// Every wait is bounded; on expiry the CTA stops issuing work, drains what it
// issued, writes NaN markers for its pieces' partials, frees TMEM and returns.

#pragma once

namespace kvq {

template <int D, int FMT>
struct PfCfg {
  static constexpr bool BF = FMT == KVQ_BF16;
  static constexpr bool F8 = FMT == KVQ_FP8_E4M3 || FMT == KVQ_FP8_E5M2;
  static constexpr bool SI = FMT == KVQ_INT8_CHANNEL;            // static per-channel / per-tensor
  static constexpr bool ZP = FMT == KVQ_INT8_ASYM;               // per-token scale + zero point
  static constexpr int E = BF ? 2 : 1;                           // bytes per cached element
  static constexpr int PAGE = kBlockSize * D * E;                // raw page bytes
  static constexpr int MV = F8 ? 1 : (ZP ? 2 : 0);               // per-token metadata values
  static constexpr int METAB = kBlockSize * MV * 2;              // raw scale bytes per page
  static constexpr int NST = 2;                                  // raw ring stages (tiles)
  static constexpr int HT = 64;                                  // tokens per half tile
  static constexpr int CPAGE = kBlockSize * D * 2;               // page bytes at 16 bits
  static constexpr int QP = SI ? 2 : 1;                          // query parts
  static constexpr int QBYTES = 128 * D * 2;                     // one query operand
  // converted half-tile stages: three let the converters run two halves ahead
  // of the PV product (static INT8 keeps two: its query takes two operands)
  static constexpr int NCS = BF ? 0 : (SI ? 2 : 3);
  static constexpr int NCB = BF ? 3 : NCS;                        // half-tile slots of the barriers
  static constexpr int CMETA = 4 * HT * 4 + 128;                 // floats a, b, sv, zv per token; max sv
  static constexpr int CSTAGE = 8 * CPAGE + CMETA;               // K (4 pages), V (4 pages), meta
  // operand strides (bytes): K pages and the query are K-major with 8-row
  // groups of 16-byte chunks; V pages are stored transposed (tokens contiguous)
  static constexpr uint32_t K_LBO = 128, K_SBO = 16 * D;          // 16-bit K page
  static constexpr uint32_t V_LBO = 16 * D, V_SBO = 128;          // 16-bit V page
  static constexpr uint32_t Q_LBO = 128, Q_SBO = 16 * D;
  // TMEM: three S / P buffers of 64 columns, then O (D columns)
  static constexpr int NSB = 3;                                  // S / P buffers in TMEM
  static constexpr int COL_S = 0, COL_O = 64 * NSB, TMEM_COLS = 512;
  // shared memory carve-up (offsets from a 1024-byte aligned base)
  static constexpr int OFF_RK = 0;                               // [NST][8 pages]
  static constexpr int OFF_RV = OFF_RK + NST * 8 * PAGE;
  static constexpr int OFF_RKM = OFF_RV + NST * 8 * PAGE;        // [NST][8][METAB]
  static constexpr int OFF_RVM = OFF_RKM + NST * 8 * (METAB > 0 ? METAB : 16);
  static constexpr int OFF_C = (OFF_RVM + NST * 8 * (METAB > 0 ? METAB : 16) + 127) / 128 * 128;
  static constexpr int OFF_Q = OFF_C + NCS * CSTAGE;             // [QP]
  static constexpr int OFF_XCH = OFF_Q + QP * QBYTES;            // float [2][2][128] maxima, [2][128][2] sums
  static constexpr int OFF_BAR = OFF_XCH + (2 * 2 * 128 + 2 * 128 * 2) * 4;
  static constexpr int NBAR = 2 * NST + 2 * NCB + 3 * NSB + 3;  // rfull/rfree, cfull/cfree, sfull/pready/pvdone, q, ofree, drain
  static constexpr int OFF_MASK = (OFF_BAR + 8 * NBAR + 15) / 16 * 16;   // uint32 [NST] raw, [NCB] conv
  static constexpr int OFF_RED = (OFF_MASK + 4 * (NST + NCB) + 15) / 16 * 16;   // long long [8] prologue
  static constexpr int OFF_MISC = OFF_RED + 128;                 // tmem base, abort flag, start (b, P)
  static constexpr int SMEM = OFF_MISC + 32 + 1024;              // + alignment slack
  static_assert(OFF_RKM % 16 == 0 && OFF_C % 128 == 0 && OFF_Q % 128 == 0 && OFF_BAR % 8 == 0,
                "smem alignment");
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

// Two E4M3 (or E5M2) codes per 16-bit half of `w` -> two packed f16x2 words.
template <bool E4>
__device__ __forceinline__ void fp8x4_to_f16x4(uint32_t w, uint32_t& lo, uint32_t& hi) {
  if constexpr (E4)
    asm("{\n\t.reg .b16 a, b;\n\tmov.b32 {a, b}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, a;\n\tcvt.rn.f16x2.e4m3x2 %1, b;\n\t}\n"
        : "=r"(lo), "=r"(hi) : "r"(w));
  else
    asm("{\n\t.reg .b16 a, b;\n\tmov.b32 {a, b}, %2;\n\t"
        "cvt.rn.f16x2.e5m2x2 %0, a;\n\tcvt.rn.f16x2.e5m2x2 %1, b;\n\t}\n"
        : "=r"(lo), "=r"(hi) : "r"(w));
}

// Four int8 codes -> two packed f16x2 words (exact): 1024 + (c + 128) is
// built by a byte permute and 1152 subtracted.
__device__ __forceinline__ void s8x4_to_f16x4(uint32_t w, uint32_t& lo, uint32_t& hi) {
  const uint32_t x = w ^ 0x80808080u;
  const uint32_t p0 = __byte_perm(x, 0x64646464u, 0x4140);
  const uint32_t p1 = __byte_perm(x, 0x64646464u, 0x4342);
  const __half2 off = __halves2half2(__ushort_as_half(0x6480), __ushort_as_half(0x6480));   // 1152
  const __half2 h0 = __hsub2(*reinterpret_cast<const __half2*>(&p0), off);
  const __half2 h1 = __hsub2(*reinterpret_cast<const __half2*>(&p1), off);
  lo = *reinterpret_cast<const uint32_t*>(&h0);
  hi = *reinterpret_cast<const uint32_t*>(&h1);
}

// 2^x by the hardware approximation (relative error about 2^-22; results below
// 2^-126 flush to 0, 2^-inf = 0).
__device__ __forceinline__ float ex2_ftz(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 16 codes (one 16-byte chunk) -> 16 f16 values (32 bytes), little-endian.
template <int FMT>
__device__ __forceinline__ void codes16_to_f16(const uint4 c, uint4& o0, uint4& o1) {
  const uint32_t w[4] = {c.x, c.y, c.z, c.w};
  uint32_t r[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if constexpr (FMT == KVQ_FP8_E4M3) fp8x4_to_f16x4<true>(w[i], r[2 * i], r[2 * i + 1]);
    else if constexpr (FMT == KVQ_FP8_E5M2) fp8x4_to_f16x4<false>(w[i], r[2 * i], r[2 * i + 1]);
    else s8x4_to_f16x4(w[i], r[2 * i], r[2 * i + 1]);
  }
  o0 = make_uint4(r[0], r[1], r[2], r[3]);
  o1 = make_uint4(r[4], r[5], r[6], r[7]);
}

// The row of `x` (BF16 pairs) as the f16 or bf16 operand row: BF16 passes
// through; f16 takes x * 2^e (exact unless an element is below 2^-14 after
// the scaling, i.e. 2^-29 of the row's largest).
__device__ __forceinline__ uint32_t bf16x2_to_f16x2_scaled(uint32_t w, float up) {
  const __half2 h = __floats2half2_rn(bf16_lo(w) * up, bf16_hi(w) * up);
  return *reinterpret_cast<const uint32_t*>(&h);
}

template <int D, int FMT>
__global__ void __launch_bounds__(448, 1) prefill_mma_kernel(
    const __nv_bfloat16* __restrict__ q, const uint8_t* __restrict__ kc,
    const uint8_t* __restrict__ vc, const __nv_bfloat16* __restrict__ ks,
    const __nv_bfloat16* __restrict__ vs, const int32_t* __restrict__ tables,
    const int32_t* __restrict__ ctx_lens, int B, int Hk, int G, int nq, int nrb, int NB, int W,
    int max_ctx, int unit_tiles, int slots, float qk_scale, int per_tensor, long long wait_limit,
    float* __restrict__ part_o, float* __restrict__ part_ml, int32_t* __restrict__ part_cnt) {
  using C = PfCfg<D, FMT>;
  using namespace tc;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int NWARPS = 14;
  const int R = G * nq;                                    // query rows of a KV head
  const int rb = int(blockIdx.x % nrb);                    // this CTA's row block
  const long long grp = blockIdx.x / nrb, NG = gridDim.x / nrb;

  uint8_t* rk = smem + C::OFF_RK;
  uint8_t* rv = smem + C::OFF_RV;
  uint8_t* rkm = smem + C::OFF_RKM;
  uint8_t* rvm = smem + C::OFF_RVM;
  uint8_t* cst = smem + C::OFF_C;
  uint8_t* qop = smem + C::OFF_Q;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* rfull = bars;                   // [NST] producer -> converters / MMA
  uint64_t* rfree = bars + C::NST;          // [NST]
  uint64_t* cfull = bars + 2 * C::NST;      // [NCB] converters -> MMA, softmax
  uint64_t* cfree = cfull + C::NCB;         // [NCB] a converted stage's PV product has completed
  uint64_t* sfull = cfree + C::NCB;         // [NSB] S of a half tile in TMEM
  uint64_t* pready = sfull + C::NSB;        // [NSB] P' of a half tile in TMEM
  uint64_t* pvdone = pready + C::NSB;       // [NSB] PV of a half tile complete
  uint64_t* qready = pvdone + C::NSB;       // the query operand of the next piece
  uint64_t* ofree = qready + 1;             // O of the last piece read
  uint64_t* drain = ofree + 1;
  volatile uint32_t* rmask = reinterpret_cast<volatile uint32_t*>(smem + C::OFF_MASK);   // [NST]
  volatile uint32_t* cmask = rmask + C::NST;                                            // [NCB]
  long long* red64 = reinterpret_cast<long long*>(smem + C::OFF_RED);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  int* misci = reinterpret_cast<int*>(smem + C::OFF_MISC + 8);
  long long* miscll = reinterpret_cast<long long*>(smem + C::OFF_MISC + 16);

  // ------------------------------------------------------------ set-up
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NST; ++s) {
      mbar_init(rfull + s, 1);
      mbar_init(rfree + s, C::BF ? 1 : 128);
    }
    for (int j = 0; j < C::NCB; ++j) {
      mbar_init(cfull + j, 128);
      mbar_init(cfree + j, 1);
    }
    for (int j = 0; j < C::NSB; ++j) {
      mbar_init(sfull + j, 1);
      mbar_init(pready + j, 256);
      mbar_init(pvdone + j, 1);
    }
    mbar_init(qready, 256);
    mbar_init(ofree, 256);
    mbar_init(drain, 1);
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // the set-up above touches no global memory; every argument in device memory
  // is read after the kernel ahead on the stream has finished
  grid_dep_wait();
  grid_dep_launch_dependents();

  // ------------------------------------------------------------ the share
  {
    long long tsum = 0;
    for (int bb = threadIdx.x; bb < B; bb += blockDim.x) {
      const int c = ctx_lens[bb];
      if (c < 0 || c > max_ctx || int64_t(c) > int64_t(W) * kBlockSize) {
        if (blockIdx.x == 0) flag_error(KVQ_DEVERR_CONTEXT);
      } else if (c > 0) {
        tsum += (c + 127) / 128 + kPieceCost;
      }
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
  const long long N = ll_min(NG, ll_max(1, T / max(1, unit_tiles)));
  if (T == 0 || grp >= N) {                                // uniform for the CTA
    if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
    return;
  }
  const long long start = (grp * T) / N;
  const long long end = ((grp + 1) * T) / N;
  {
    // the sequence holding cost position `start`: block-wide scan of run costs
    if (threadIdx.x == 0) misci[0] = -1;
    __syncthreads();
    long long run = 0;
    for (int base = 0; base < B; base += blockDim.x) {
      const int bb = base + threadIdx.x;
      int tb = bb < B ? (mma_seq_ctx(ctx_lens, bb, max_ctx, W) + 127) / 128 : 0;
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
      if (misci[0] >= 0) break;                                 // uniform
    }
  }
  const int b0 = misci[0];
  const long long P0 = miscll[0];
  auto cta_of = [&](long long x) -> long long { return ((x + 1) * N - 1) / T; };

  PieceWalk walk;
  walk.init(b0, P0, start, end, Hk, ctx_lens, B, max_ctx, W);

  if (warp == 0) {
    // ---------------------------------------------------------- producer
    const uint64_t pol = l2_evict_first_policy();
    const int p8 = lane & 7;
    constexpr int CPP = C::METAB > 0 ? C::METAB / 16 : 1;    // 16-byte scale chunks per page
    const int sp = lane / CPP, sc = lane % CPP;
    // block id of page p8 of tile `tile` of `pw` (-2: no page there)
    auto load_id = [&](const PieceWalk& pw, int tile) -> int {
      if (lane >= 8 || pw.done) return -2;
      const int tok0 = tile * 128;
      const int npg = min(8, (pw.ctx - tok0 + kBlockSize - 1) / kBlockSize);
      return p8 < npg ? tables[int64_t(pw.b) * W + tok0 / kBlockSize + p8] : -2;
    };
    auto step = [&](PieceWalk& pw, int& tile) {
      if (pw.done) return;
      if (++tile >= pw.hi) {
        pw.next(Hk, ctx_lens, B, max_ctx, W);
        tile = pw.lo;
      }
    };
    PieceWalk c0 = walk, c1 = walk;
    int i0 = walk.lo, i1 = walk.lo;
    step(c1, i1);
    int id0 = load_id(c0, i0);
    bool iss[C::NST];
    uint32_t par[C::NST];
#pragma unroll
    for (int s = 0; s < C::NST; ++s) { iss[s] = false; par[s] = 0; }
    for (int gt = 0; !c0.done; ++gt) {
      const int s = gt % C::NST;
      const uint32_t ph = (gt / C::NST) & 1;
      const int id1 = load_id(c1, i1);                     // next tile's block ids, in flight
      const int h = c0.h;
      if (lane < 8 && id0 != -2 && (id0 < 0 || id0 >= NB)) flag_error(KVQ_DEVERR_BLOCK);
      const bool valid = lane < 8 && id0 >= 0 && id0 < NB;
      const uint32_t mask = __ballot_sync(0xffffffffu, valid) & 0xFFu;
      const int blk = __shfl_sync(0xffffffffu, id0, p8);
      const bool mine = ((mask >> p8) & 1u) != 0u;
      const int64_t page = int64_t(blk) * Hk + h;
      uint4 kv = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
      const bool smine = C::MV > 0 && sp < 8 && ((mask >> (sp & 7)) & 1u) != 0u;
      if constexpr (C::MV > 0) {
        const int sblk = __shfl_sync(0xffffffffu, id0, sp & 7);
        if (smine) {
          const int64_t off = (int64_t(sblk) * Hk + h) * C::METAB + sc * 16;
          kv = __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(ks) + off));
          vv = __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(vs) + off));
        }
      }
      bool ok = true;
      if (lane == 0) {
        ok = mbar_wait(rfree + s, ph ^ 1, abort_flag, wait_limit);
        if (ok) mbar_expect_tx(rfull + s, 2u * uint32_t(__popc(mask)) * uint32_t(C::PAGE));
      }
      if (!__shfl_sync(0xffffffffu, int(ok), 0)) break;
      if (lane < 8 && mine) {
        bulk_g2s(rk + (s * 8 + p8) * C::PAGE, kc + page * C::PAGE, C::PAGE, rfull + s, pol);
        bulk_g2s(rv + (s * 8 + p8) * C::PAGE, vc + page * C::PAGE, C::PAGE, rfull + s, pol);
      }
      iss[s] = true;
      par[s] = ph;
      if constexpr (C::MV > 0) {
        if (smine) {
          *reinterpret_cast<uint4*>(rkm + (s * 8 + sp) * C::METAB + sc * 16) = kv;
          *reinterpret_cast<uint4*>(rvm + (s * 8 + sp) * C::METAB + sc * 16) = vv;
        }
      }
      __syncwarp();
      if (lane == 0) {
        rmask[s] = mask;
        mbar_arrive(rfull + s);
      }
      c0 = c1; i0 = i1; id0 = id1;
      step(c1, i1);
    }
    if (lane == 0 && *abort_flag) {
      // let the copies already issued land before the CTA's smem goes away
      volatile int no_abort = 0;
      for (int s = 0; s < C::NST; ++s)
        if (iss[s]) mbar_wait(rfull + s, par[s], &no_abort, kMmaWaitLimitCycles);
    }
  } else if (warp >= 10) {
    // ---------------------------------------------------------- converters
    const int ct = threadIdx.x - 320;                      // 0..127
    const float c0 = qk_scale;                             // sm_scale * log2(e): base-2 scores
    bool ok = true;
    int gt = 0, u = 0;
    for (PieceWalk pw = walk; !pw.done; pw.next(Hk, ctx_lens, B, max_ctx, W)) {
      for (int i = pw.lo; i < pw.hi; ++i, ++gt) {
        const int s = gt % C::NST;
        if (ok) ok = mbar_wait(rfull + s, (gt / C::NST) & 1, abort_flag, wait_limit);
        const uint32_t pm = rmask[s];
        for (int hh = 0; hh < 2; ++hh, ++u) {
          const int cs = u % C::NCB;
          // the stage (and its page mask) of half u - NCB is free once that
          // half's PV product has completed
          if (ok && u >= C::NCB) ok = mbar_wait(cfree + cs, (u / C::NCB - 1) & 1, abort_flag, wait_limit);
          const int tok0 = i * 128 + hh * 64;              // first token of the half
          // tokens of page p of the half that hold cache entries (0 for an
          // invalid page)
          auto nvalid = [&](int p) -> int {
            if (((pm >> (4 * hh + p)) & 1u) == 0u) return 0;
            return max(0, min(16, pw.ctx - (tok0 + 16 * p)));
          };
          if (ok) {
            if constexpr (C::BF) {
              // zero the V entries of tokens past the end (and of invalid pages)
              for (int p = 0; p < 4; ++p) {
                const int nv = nvalid(p);
                if (nv == 16) continue;                    // uniform
                uint8_t* pg = rv + (s * 8 + 4 * hh + p) * C::PAGE;
                for (int x = ct; x < 2 * D; x += 128) {
                  const int uu = x / D;                    // tokens 8 uu .. 8 uu + 7
                  uint4* ch = reinterpret_cast<uint4*>(pg + x * 16);
                  const int keep = max(0, min(8, nv - 8 * uu));
                  if (keep == 8) continue;
                  uint32_t w[4] = {ch->x, ch->y, ch->z, ch->w};
#pragma unroll
                  for (int e = 0; e < 4; ++e) {
                    const uint32_t m = (2 * e < keep ? 0x0000FFFFu : 0u) | (2 * e + 1 < keep ? 0xFFFF0000u : 0u);
                    w[e] &= m;
                  }
                  *ch = make_uint4(w[0], w[1], w[2], w[3]);
                }
              }
            } else {
              uint8_t* cb = cst + cs * C::CSTAGE;
              uint8_t* ck = cb;
              uint8_t* cv = cb + 4 * C::CPAGE;
              float* cm = reinterpret_cast<float*>(cb + 8 * C::CPAGE);
              // every raw chunk of the half is loaded before any converted one is
              // stored (the stores could alias the loads as far as the compiler
              // knows, which would serialize them)
              constexpr int NIT = 4 * D / 128;
              const uint8_t* rkh = rk + (s * 8 + 4 * hh) * C::PAGE;
              const uint8_t* rvh = rv + (s * 8 + 4 * hh) * C::PAGE;
              uint4 kraw[NIT], vraw[NIT];
#pragma unroll
              for (int it = 0; it < NIT; ++it) {
                // K: raw 16-byte chunk k of a page holds 16 channels of one token;
                // V: raw chunk d holds 16 tokens of channel d (in page units the
                // two are the same byte offset)
                const int x = ct + 128 * it;
                kraw[it] = *reinterpret_cast<const uint4*>(rkh + (x / D) * C::PAGE + (x % D) * 16);
                vraw[it] = *reinterpret_cast<const uint4*>(rvh + (x / D) * C::PAGE + (x % D) * 16);
              }
#pragma unroll
              for (int it = 0; it < NIT; ++it) {
                const int x = ct + 128 * it;
                const int p = x / D, k = x % D;
                const int g = k / (D / 2), rem = k % (D / 2), c = rem >> 3, tt = rem & 7;
                uint4 o0, o1;
                codes16_to_f16<FMT>(kraw[it], o0, o1);
                uint8_t* dst = ck + p * C::CPAGE + g * 16 * D + (2 * c) * 128 + tt * 16;
                *reinterpret_cast<uint4*>(dst) = o0;
                *reinterpret_cast<uint4*>(dst + 128) = o1;
              }
              // V (64 | D: the page, hence nv, is the same for every thread of a
              // warp)
#pragma unroll
              for (int it = 0; it < NIT; ++it) {
                const int x = ct + 128 * it;
                const int p = x / D, d = x % D;
                const int nv = nvalid(p);
                uint4 o0, o1;
                codes16_to_f16<FMT>(vraw[it], o0, o1);
                uint32_t w[8] = {o0.x, o0.y, o0.z, o0.w, o1.x, o1.y, o1.z, o1.w};
                if (nv < 16) {
#pragma unroll
                  for (int e = 0; e < 8; ++e)
                    w[e] &= (2 * e < nv ? 0x0000FFFFu : 0u) | (2 * e + 1 < nv ? 0xFFFF0000u : 0u);
                }
                uint8_t* pg = cv + p * C::CPAGE;
                *reinterpret_cast<uint4*>(pg + d * 16) = make_uint4(w[0], w[1], w[2], w[3]);
                *reinterpret_cast<uint4*>(pg + (D + d) * 16) = make_uint4(w[4], w[5], w[6], w[7]);
              }
              // per-token column factors: score = S a + b qsum, P' = p sv, V zero
              // point zv (threads 0..63, one token each)
              if (ct < C::HT) {
                const int p = ct >> 4, tk = ct & 15;
                const bool tv = tk < nvalid(p);
                float a = 0.f, b = 0.f, sv = 0.f, zv = 0.f;
                if (tv) {
                  if constexpr (C::F8) {
                    const int o = (s * 8 + 4 * hh + p) * C::METAB + tk * 2;
                    a = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(rkm + o)) * c0;
                    sv = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(rvm + o));
                  } else if constexpr (C::ZP) {
                    const int o = (s * 8 + 4 * hh + p) * C::METAB + tk * 4;
                    const __nv_bfloat162 km = *reinterpret_cast<const __nv_bfloat162*>(rkm + o);
                    const __nv_bfloat162 vm = *reinterpret_cast<const __nv_bfloat162*>(rvm + o);
                    a = __low2float(km) * c0;
                    b = -__low2float(km) * __high2float(km) * c0;
                    sv = __low2float(vm);
                    zv = __high2float(vm);
                  } else {
                    a = c0;
                    sv = 1.f;
                  }
                }
                cm[ct] = a;
                cm[C::HT + ct] = b;
                cm[2 * C::HT + ct] = sv;
                cm[3 * C::HT + ct] = zv;
                const float svw = warp_max(sv);              // V scales are >= 0
                if ((ct & 31) == 0) cm[4 * C::HT + (ct >> 5)] = svw;
              }
            }
            fence_proxy_async_smem();
          }
          if (ct == 0) cmask[cs] = (pm >> (4 * hh)) & 0xFu;
          mbar_arrive(cfull + cs);
        }
        if constexpr (!C::BF) mbar_arrive(rfree + s);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_s = idesc_f16(C::HT, C::BF);   // Q x K^T: f16 (bf16 for a BF16 cache)
      constexpr uint32_t id_pv = idesc_f16(D, C::BF);       // P' x V: f16 (bf16 for a BF16 cache)
      const uint32_t qaddr = smem_u32(qop), rkaddr = smem_u32(rk), rvaddr = smem_u32(rv);
      const uint32_t caddr = smem_u32(cst);
      bool ok = true;
      int u = 0, gt = 0, pc = 0;
      // the half tile whose PV product is pending
      int pend = -1, pend_s = 0, pend_hh = 0, pend_pc = 0;
      bool pend_first = false;
      auto issue_pv = [&]() -> bool {
        const int cs = pend % C::NSB, ck = pend % C::NCB;
        if (!mbar_wait(pready + cs, (pend / C::NSB) & 1, abort_flag, wait_limit)) return false;
        // a piece's first product overwrites O: the softmax warps have read the last piece's
        if (pend_first && pend_pc > 0 && !mbar_wait(ofree, (pend_pc - 1) & 1, abort_flag, wait_limit))
          return false;
        tc_fence_after();
        const uint32_t vb = C::BF ? rvaddr + (pend_s * 8 + 4 * pend_hh) * C::PAGE
                                  : caddr + ck * C::CSTAGE + 4 * C::CPAGE;
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
          for (int kk = 0; kk < C::HT / 16; ++kk)
            mma_f16_ts(tmem + C::COL_O, tmem + C::COL_S + cs * 64 + j * 32 + 8 * kk,
                       sdesc_plain(vb + kk * C::CPAGE, C::V_LBO, C::V_SBO), id_pv,
                       (pend_first && j == 0 && kk == 0) ? 0u : 1u);
        mma_commit(pvdone + cs);
        mma_commit(cfree + ck);
        if (C::BF && pend_hh == 1) mma_commit(rfree + pend_s);    // the raw stage is consumed
        return true;
      };
      for (PieceWalk pw = walk; ok && !pw.done; pw.next(Hk, ctx_lens, B, max_ctx, W), ++pc) {
        ok = mbar_wait(qready, pc & 1, abort_flag, wait_limit);
        if (!ok) break;
        tc_fence_after();
        for (int i = pw.lo; ok && i < pw.hi; ++i, ++gt) {
          const int s = gt % C::NST;
          for (int hh = 0; hh < 2; ++hh, ++u) {
            const int cs = u % C::NSB, ck = u % C::NCB;
            // the half's K operand is ready; its S / P columns are free once the
            // PV product of half u - NSB has completed
            ok = mbar_wait(cfull + ck, (u / C::NCB) & 1, abort_flag, wait_limit) &&
                 (u < C::NSB || mbar_wait(pvdone + cs, (u / C::NSB - 1) & 1, abort_flag, wait_limit));
            if (!ok) break;
            tc_fence_after();
            const uint32_t kb = C::BF ? rkaddr + (s * 8 + 4 * hh) * C::PAGE : caddr + ck * C::CSTAGE;
#pragma unroll
            for (int qp = 0; qp < C::QP; ++qp)
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk)
                mma_ss<0>(tmem + C::COL_S + cs * 64,
                          sdesc_plain(qaddr + qp * C::QBYTES + kk * 256, C::Q_LBO, C::Q_SBO),
                          sdesc_plain(kb + kk * 256, C::K_LBO, C::K_SBO), id_s,
                          (qp | kk) ? 1u : 0u);
            mma_commit(sfull + cs);
            if (pend >= 0) {
              ok = issue_pv();
              if (!ok) break;
            }
            pend = u;
            pend_s = s;
            pend_hh = hh;
            pend_first = i == pw.lo && hh == 0;
            pend_pc = pc;
          }
        }
      }
      if (ok && pend >= 0) issue_pv();
      // every MMA issued so far completes before TMEM is released
      volatile int no_abort = 0;
      mma_commit(drain);
      mbar_wait(drain, 0, &no_abort, kMmaWaitLimitCycles);
    }
  } else {
    // ---------------------------------------------------------- softmax warps
    const int quarter = warp & 3;
    const int set = (warp - 2) >> 2;                      // columns [32 set, 32 set + 32) of a half
    const int r = quarter * 32 + lane;                    // query row of the block, TMEM lane
    constexpr int HC = C::HT / 2;                         // columns per thread and half
    float* xmax = reinterpret_cast<float*>(smem + C::OFF_XCH);          // [2][2][128]
    float2* xsum = reinterpret_cast<float2*>(smem + C::OFF_XCH + 2 * 2 * 128 * 4);   // [2][128]
    const int pair_bar = 2 + quarter;                     // the two warps of this lane quarter
    const uint32_t lane_base = uint32_t(quarter * 32) << 16;
    const int rho = rb * 128 + r;                         // row of the KV head: g * nq + j
    const bool row_ok = rho < R;
    const int jpos = row_ok ? rho % nq : 0;               // chunk position of the row
    bool ok = true;
    // tcgen05.ld / st are warp-wide: every lane of a warp takes the same path
    auto wait_all = [&](uint64_t* bar, uint32_t parity) {
      if (ok) ok = mbar_wait(bar, parity, abort_flag, wait_limit);
      ok = __all_sync(0xffffffffu, ok);
    };

    // a pair of P' parts in the PV product's operand type
    struct P16 {
      uint32_t bits;
      __device__ __forceinline__ static P16 make(float a, float b) {
        P16 r;
        if constexpr (C::BF) {
          const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
          r.bits = *reinterpret_cast<const uint32_t*>(&v);
        } else {
          const __half2 v = __floats2half2_rn(a, b);
          r.bits = *reinterpret_cast<const uint32_t*>(&v);
        }
        return r;
      }
      __device__ __forceinline__ float2 f2() const {
        if constexpr (C::BF) return make_float2(bf16_lo(bits), bf16_hi(bits));
        const __half2 v = *reinterpret_cast<const __half2*>(&bits);
        return __half22float2(v);
      }
    };
    // The query row of a piece into the query operand (K-major 8-row groups of
    // 16-byte chunks), once per piece (a piece spans many tiles): the row is
    // streamed from global memory 8 channels at a time, twice (its largest
    // element first), in rolled loops that keep the kernel's code small.
    // Returns the factor that takes S back to the row's units and, through
    // qsum, the sum of the operand's values (the zero-point term). Both warp
    // sets compute the factors; set 0 writes the operand.
    auto store_q = [&](const PieceWalk& pw, float& down, float& qsum) {
      down = 1.f;
      qsum = 0.f;
      const bool wr = set == 0;
      const bool have = !pw.done && row_ok;
      const uint4* src = reinterpret_cast<const uint4*>(q + ((int64_t(pw.b) * Hk + pw.h) * R + rho) * D);
      uint8_t* row = qop + (r >> 3) * C::Q_SBO + (r & 7) * 16;
      auto chunk = [&](int c) -> uint4 { return have ? src[c] : make_uint4(0, 0, 0, 0); };
      // x = q (static INT8: q times the K scale of the channel)
      auto xval = [&](uint32_t w, int half, int d) -> float {
        float x = half ? bf16_hi(w) : bf16_lo(w);
        if constexpr (C::SI) x *= __bfloat162float(ks[per_tensor ? 0 : pw.h * D + d]);
        return x;
      };
      if constexpr (C::BF) {
        if (wr) {
#pragma unroll 2
          for (int c = 0; c < D / 8; ++c) *reinterpret_cast<uint4*>(row + c * C::Q_LBO) = chunk(c);
        }
      } else {
        float amax = 0.f;
#pragma unroll 2
        for (int c = 0; c < D / 8; ++c) {
          const uint4 u4 = chunk(c);
          const uint32_t w[4] = {u4.x, u4.y, u4.z, u4.w};
#pragma unroll
          for (int k = 0; k < 8; ++k) amax = fmaxf(amax, fabsf(xval(w[k >> 1], k & 1, 8 * c + k)));
        }
        // power-of-two scaling: the largest element lands in [2^14, 2^15)
        int e = 0;
        if (amax > 0.f) e = 14 - ilogbf(amax);
        e = max(-100, min(100, e));
        const float up = __int_as_float((127 + e) << 23);
        down = __int_as_float((127 - e) << 23);
#pragma unroll 1
        for (int c = 0; c < D / 8; ++c) {
          const uint4 u4 = chunk(c);
          const uint32_t w[4] = {u4.x, u4.y, u4.z, u4.w};
          uint32_t hi[4], lo[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float a = xval(w[k], 0, 8 * c + 2 * k) * up, b = xval(w[k], 1, 8 * c + 2 * k + 1) * up;
            const __half2 h = __floats2half2_rn(a, b);
            hi[k] = *reinterpret_cast<const uint32_t*>(&h);
            if constexpr (C::SI) {
              const __half2 l2 = __floats2half2_rn(a - __low2float(h), b - __high2float(h));
              lo[k] = *reinterpret_cast<const uint32_t*>(&l2);
            }
            if constexpr (C::ZP) qsum += __low2float(h) + __high2float(h);
          }
          if (wr) {
            *reinterpret_cast<uint4*>(row + c * C::Q_LBO) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
            if constexpr (C::SI)
              *reinterpret_cast<uint4*>(row + C::QBYTES + c * C::Q_LBO) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
          }
        }
      }
      fence_proxy_async_smem();
    };

    float down = 1.f, qsum = 0.f, down_n = 1.f, qsum_n = 0.f;
    store_q(walk, down, qsum);
    mbar_arrive(qready);

    int u = 0;
    for (PieceWalk pw = walk; !pw.done;) {
      PieceWalk nxt = pw;
      nxt.next(Hk, ctx_lens, B, max_ctx, W);
      const int slot = int(grp - cta_of(pw.first_tile(Hk)));
      const bool last = pw.hi == pw.nt;
      // tokens t < lim are attended: the chunk's position j sees the context
      // up to and including its own token
      const int lim = row_ok ? max(0, pw.ctx - nq + 1 + jpos) : 0;
      float m_run = -INFINITY, l = 0.f, corr = 0.f;
      for (int i = pw.lo; i < pw.hi; ++i) {
        for (int hh = 0; hh < 2; ++hh, ++u) {
          const int cs = u % C::NSB, ck = u % C::NCB;      // TMEM buffer, converted stage
          wait_all(cfull + ck, (u / C::NCB) & 1);
          wait_all(sfull + cs, (u / C::NSB) & 1);
          tc_fence_after();
          if (i == pw.hi - 1 && hh == 1 && !nxt.done) {
            // every S product of this piece has completed: the next piece's
            // query may replace this one
            store_q(nxt, down_n, qsum_n);
            mbar_arrive(qready);
          }
          uint32_t sr[HC];
          if (ok) {
#pragma unroll
            for (int c = 0; c < HC / 16; ++c)
              tmem_ld16(tmem + lane_base + C::COL_S + cs * 64 + HC * set + 16 * c,
                        *reinterpret_cast<uint32_t(*)[16]>(sr + 16 * c));
            tmem_ld_wait();
          } else {
#pragma unroll
            for (int c = 0; c < HC; ++c) sr[c] = 0u;
          }
          const float* cm = reinterpret_cast<const float*>(cst + ck * C::CSTAGE + 8 * C::CPAGE);
          const uint32_t pmh = cmask[ck];
          const int t0 = i * 128 + hh * 64 + HC * set;    // first token of this thread's columns
          // scores in the operand's units (x * down is the base-2 score), two
          // columns per instruction, in place of S; columns are masked only in
          // the halves where some row of the warp needs it
          const bool full = __all_sync(0xffffffffu, t0 + HC <= lim && pmh == 0xFu);
          float2* x2 = reinterpret_cast<float2*>(sr);
          const float2* a2 = reinterpret_cast<const float2*>(cm + HC * set);
          const float2* b2 = reinterpret_cast<const float2*>(cm + C::HT + HC * set);
          const float2 qs2 = make_float2(qsum, qsum), k2 = make_float2(qk_scale, qk_scale);
          float2 mx = make_float2(-INFINITY, -INFINITY);
#pragma unroll
          for (int k = 0; k < HC / 2; ++k) {
            const float2 sv_ = make_float2(__uint_as_float(sr[2 * k]), __uint_as_float(sr[2 * k + 1]));
            float2 x;
            if constexpr (C::BF) x = __fmul2_rn(sv_, k2);
            else if constexpr (C::ZP) x = __ffma2_rn(sv_, a2[k], __fmul2_rn(b2[k], qs2));
            else x = __fmul2_rn(sv_, a2[k]);
            if (!full) {
              const int c = 2 * k;
              const bool pg = ((pmh >> ((HC * set + c) >> 4)) & 1u) != 0u;
              if (!(pg && t0 + c < lim)) x.x = -INFINITY;
              if (!(pg && t0 + c + 1 < lim)) x.y = -INFINITY;
            }
            x2[k] = x;
            mx.x = fmaxf(mx.x, x.x);
            mx.y = fmaxf(mx.y, x.y);
          }
          float mt = fmaxf(mx.x, mx.y);
          // the row maximum over both warps' columns (double-buffered by half)
          xmax[((u & 1) * 2 + set) * 128 + r] = mt;
          named_bar_sync(pair_bar, 64);
          mt = fmaxf(mt, xmax[((u & 1) * 2 + (set ^ 1)) * 128 + r]);
          mt *= down;
          // the largest weight of the half is at most 2^(mt - m_run) * svmax: the
          // reference moves with log2(svmax) too, so that P' stays below 2^8 and
          // its f16 parts keep their precision whatever the V scales are (a
          // zero largest scale counts as 2^-64: its tokens still count in l)
          if constexpr (C::F8 || C::ZP) {
            const float svm = fmaxf(cm[4 * C::HT], cm[4 * C::HT + 1]);
            mt += svm > 0.f ? fmaxf(__log2f(svm), -64.f) : -64.f;
          }
          // lazy rescaling: the reference moves only when the largest weight
          // would exceed 2^8 relative to it; O (this piece's earlier halves:
          // their PV products are waited for only then) is rescaled in TMEM by
          // the whole warp, with factor 1 for rows that keep their reference
          float alpha = 1.f;
          if (mt > m_run + 8.f) {
            if (m_run != -INFINITY) {
              alpha = exp2f(m_run - mt);
              l *= alpha;
              corr *= alpha;
            }
            m_run = mt;
          }
          if (__any_sync(0xffffffffu, alpha != 1.f)) {
            if (u >= 1) wait_all(pvdone + ((u - 1) % C::NSB), ((u - 1) / C::NSB) & 1);
            tc_fence_after();
          }
          if (ok && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
              const uint32_t col = C::COL_O + (D / 2) * set + 16 * c;
              uint32_t ov[16];
              tmem_ld16(tmem + lane_base + col, ov);
              tmem_ld_wait();
#pragma unroll
              for (int e = 0; e < 16; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
              tmem_st16(tmem + lane_base + col, ov);
            }
            tmem_st_wait();
          }
          // P' = p * v_scale as two 16-bit parts, token pairs per word, written
          // to TMEM 32 tokens at a time
          const bool any = m_run != -INFINITY;
          const float2 dn2 = make_float2(down, down), nm2 = make_float2(-m_run, -m_run);
          const float2 m1 = make_float2(-1.f, -1.f);
          const float2* sv2 = reinterpret_cast<const float2*>(cm + 2 * C::HT + HC * set);
          const float2* zv2 = reinterpret_cast<const float2*>(cm + 3 * C::HT + HC * set);
          float2 ls2 = make_float2(0.f, 0.f), cz2 = make_float2(0.f, 0.f);
          {
            uint32_t ph[16], pl[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) {
              const int kk = k;                             // column pair of this thread
              const float2 e = __ffma2_rn(x2[kk], dn2, nm2);
              const float2 p2 = any ? make_float2(ex2_ftz(e.x), ex2_ftz(e.y)) : make_float2(0.f, 0.f);
              ls2 = __fadd2_rn(ls2, p2);
              float2 w = p2;
              if constexpr (C::F8 || C::ZP) w = __fmul2_rn(p2, sv2[kk]);
              P16 hv = P16::make(w.x, w.y);
              const float2 hf = hv.f2();
              const float2 rr = __ffma2_rn(hf, m1, w);      // w - hi, exact
              P16 lv = P16::make(rr.x, rr.y);
              ph[k] = hv.bits;
              pl[k] = lv.bits;
              if constexpr (C::ZP)
                cz2 = __ffma2_rn(__fadd2_rn(hf, lv.f2()), zv2[kk], cz2);
            }
            if (ok) {
              tmem_st16(tmem + lane_base + C::COL_S + cs * 64 + 16 * set, ph);
              tmem_st16(tmem + lane_base + C::COL_S + cs * 64 + 32 + 16 * set, pl);
            }
          }
          const float ls = ls2.x + ls2.y, cz = cz2.x + cz2.y;
          l += ls;
          corr += cz;
          if (ok) tmem_st_wait();
          tc_fence_before();
          mbar_arrive(pready + cs);
        }
      }

      // ---- piece partial: O of the last half, less the V zero-point term
      wait_all(pvdone + ((u - 1) % C::NSB), ((u - 1) / C::NSB) & 1);
      tc_fence_after();
      const bool good = __all_sync(0xffffffffu, ok && !*abort_flag);
      // the row's sums over both warps' columns
      xsum[set * 128 + r] = make_float2(l, corr);
      named_bar_sync(pair_bar, 64);
      {
        const float2 o2 = xsum[(set ^ 1) * 128 + r];
        l += o2.x;
        corr += o2.y;
      }
      const int64_t grow = (int64_t(pw.b) * Hk + pw.h) * R + rho;   // output row
      float* po = part_o + (grow * slots + slot) * D + (D / 2) * set;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t ov[16];
        if (good) {
          tmem_ld16(tmem + lane_base + C::COL_O + (D / 2) * set + 16 * c, ov);
          tmem_ld_wait();
        }
        if (row_ok) {
          float o[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            float x = good ? __uint_as_float(ov[e]) - corr : __int_as_float(0x7fc00000);
            if constexpr (C::SI) {
              if (good) x *= __bfloat162float(vs[per_tensor ? 0 : pw.h * D + (D / 2) * set + 16 * c + e]);
            }
            o[e] = x;
          }
#pragma unroll
          for (int e = 0; e < 16; e += 4)
            *reinterpret_cast<float4*>(po + 16 * c + e) = make_float4(o[e], o[e + 1], o[e + 2], o[e + 3]);
        }
      }
      // the sums are read before the next piece overwrites them
      named_bar_sync(pair_bar, 64);
      if (row_ok && set == 0) {
        part_ml[(grow * slots + slot) * 2] = good ? m_run : INFINITY;
        part_ml[(grow * slots + slot) * 2 + 1] = good ? l : __int_as_float(0x7fc00000);
        if (last) part_cnt[grow] = slot + 1;
      }
      tc_fence_before();
      mbar_arrive(ofree);
      down = down_n;
      qsum = qsum_n;
      pw = nxt;
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

// Paged GQA decode attention with the cache codes fed to the 5th-generation
// tensor cores as they are stored: FP8 E4M3 or E5M2 codes through
// kind::f8f6f4, INT8 codes through kind::i8 (exact integer sums), BF16 through
// kind::f16. No thread dequantizes a K or V element; the per-token scales and
// zero points are applied to the small S and P tiles instead. Static INT8
// scales (one per channel, or one per cache) vary along the contraction, so
// they multiply the query before its split (K) and the finished channel sums
// (V). Multi-query decode (speculative verification, chunked prefill) runs
// the n_query positions of a query head as extra rows of its group, each with
// its causal limit. A KV head's R = G * n_query rows are taken in row groups
// of G rows (G = 1, 2, 4 or 8, the template parameter; nrg = R / G groups):
// each group is a "virtual head" of the work list that reads the KV head's
// pages; plain decode has nrg = 1. Included by kvq_kernels.cu.
//
// Work split (persistent, stream-K): the work list is every (sequence b,
// virtual head h, 128-token tile) in order of b, then h, then tile, each (b, h) run
// also costing kPieceCost units for opening and closing its piece. Each of
// the N CTA groups takes one contiguous, equal share of the total cost (N
// is cut so that a share holds at least `unit_tiles` units). A share is a few
// "pieces", a piece being the share's tiles of one (b, h); each piece ends in
// an online-softmax partial (max, sum, unnormalised output) in a workspace
// slot, and the piece holding the last tile of (b, h) records how many slots
// the merge kernel must combine. The ring of K/V stages streams across piece
// boundaries, so a CTA fills its pipeline once.
//
// 6 warps per CTA:
//   warp 0      producer: lanes 0..7 each own one page of a 128-token tile and
//               issue its 1-D bulk copy (K page, then V page) into a ring of
//               smem stages through the TMA engine. The pages' scales are
//               loaded by every lane one tile ahead and stored into the stage
//               before its arrive (as copies they would double the TMA
//               requests, whose issue rate bounds the 8-bit tile). Block ids
//               are loaded two tiles ahead.
//   warp 1      allocates TMEM; one thread issues the MMAs.
//   warps 2..5  softmax warps, one per TMEM lane quarter; thread r owns token r
//               of the tile for S and P, channel r for O. They also build the
//               query operand of each piece, loading it one piece ahead.
// Per 128-token tile:
//   S^T[tok x n] = Kcodes[tok x D] . Qp^T[D x n]    (A: K page ring, K-major;
//                  B: the query group split into exact low-precision parts)
//   softmax in FP32 registers: s = (sum of S parts) * k_scale (INT8: minus
//     zero_point * sum(q)), online max / sum per query head.
//   P[tok x n] = the weight p * v_scale * 2^e split into low-precision parts
//     (FP8: 4 E4M3 parts, INT8: 3 unsigned bytes of a 24-bit fixed-point
//     value, BF16: 3 bf16 parts), MN-major in smem.
//   O^T[ch x n] = Vcodes^T[ch x tok] . P[tok x n]    (A: V page ring, K-major)
//   O tile -> registers, parts recombined, rescaled and accumulated in FP32.
// Each MMA result sits in TMEM; S, P and O are double-buffered so the MMA of
// one tile overlaps the softmax of the next. Every byte of the K/V crosses HBM
// once for the whole query group. Every wait is bounded: on expiry the CTA sets
// KVQ_DEVERR_TIMEOUT, stops issuing work, drains what it issued, writes NaN
// markers for its pieces' partials, frees TMEM and returns.

#pragma once

#include "kvq_tc.cuh"

namespace kvq {

// Bound on the waits that drain work already issued (copies in flight, the
// last MMAs) before the CTA exits: those always complete, so this limit only
// guards against a lost completion. The pipeline waits take the launch's
// `wait_limit` (kvq_set_wait_limit; by default this same value).
constexpr long long kMmaWaitLimitCycles = 2000000000LL;   // about one second

__device__ __forceinline__ long long ll_min(long long a, long long b) { return a < b ? a : b; }
__device__ __forceinline__ long long ll_max(long long a, long long b) { return a > b ? a : b; }

__host__ __device__ constexpr int round_up16(int x) { return x < 16 ? 16 : (x + 15) / 16 * 16; }

template <int D, int G, int FMT>
struct MmaCfg {
  static constexpr bool BF = FMT == KVQ_BF16;
  static constexpr bool F8 = FMT == KVQ_FP8_E4M3 || FMT == KVQ_FP8_E5M2;   // either FP8 code
  static constexpr bool SI = FMT == KVQ_INT8_CHANNEL;           // static per-channel / per-tensor scales
  static constexpr bool I8 = FMT == KVQ_INT8_ASYM || SI;        // s8 codes
  static constexpr bool ZP = FMT == KVQ_INT8_ASYM;              // per-token scale + zero point
  static constexpr int E = BF ? 2 : 1;                         // bytes per element
  static constexpr int KIND = BF ? 0 : (F8 ? 1 : 2);           // mma_ss kind
  static constexpr int PAGE = kBlockSize * D * E;              // bytes of one (block, head) page
  static constexpr int NST = 3;                                // ring stages
  static constexpr int MV = F8 ? 1 : (ZP ? 2 : 0);            // per-token metadata values
  static constexpr int METAB = kBlockSize * MV * 2;            // scale bytes per page
  static constexpr int QPARTS = F8 ? 2 : (I8 ? 3 : 1);
  static constexpr int PPARTS = F8 ? 4 : 3;
  static constexpr int NS = round_up16(QPARTS * G);            // S columns (B rows of QK)
  static constexpr int NO = round_up16(PPARTS * G);            // O columns (B rows of PV)
  static constexpr int NSL = (QPARTS * G + 7) / 8 * 8;         // S columns read back
  static constexpr int NOL = (PPARTS * G + 7) / 8 * 8;         // O columns read back
  static_assert(NS <= 32 && NO <= 32, "query group too large");
  static constexpr int HPW = (G + 3) / 4;                      // query heads per softmax warp
  static constexpr int S_MMAS = D * E / 32;                    // K extent of one MMA: 32 bytes
  static constexpr int PV_MMAS = 128 * E / 32;
  // operand strides (bytes)
  static constexpr uint32_t K_LBO = 128, K_SBO = 8 * D * E;    // K page: [2][D*E/16][8 tok][16 B]
  static constexpr uint32_t V_LBO = 16 * D, V_SBO = 128;       // V page: [E][D][16 B]
  static constexpr uint32_t Q_SBO = 128, Q_LBO = (NS / 8) * 128;
  static constexpr int PT = 16 / E;                            // P elements per 16-byte row
  static constexpr uint32_t P_SBO = 128, P_LBO = (NO / PT) * 128;
  static constexpr int QBYTES = NS * D * E;                    // one query operand
  static constexpr int PBYTES = NO * 128 * E;                  // one P buffer
  // TMEM columns
  static constexpr int COL_S = 0, COL_O = 64, TMEM_COLS = 128;
  // shared memory carve-up (offsets from a 128-byte aligned base)
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + NST * 8 * PAGE;
  static constexpr int OFF_KM = OFF_V + NST * 8 * PAGE;
  static constexpr int OFF_VM = OFF_KM + NST * 8 * METAB;
  static constexpr int OFF_Q = (OFF_VM + NST * 8 * METAB + 127) / 128 * 128;
  static constexpr int OFF_P = OFF_Q + QBYTES;                                  // [2]
  static constexpr int OFF_BAR = OFF_P + 2 * PBYTES;
  static constexpr int NBAR = 4 * NST + 12 + 1;
  static constexpr int OFF_RED = (OFF_BAR + 8 * NBAR + 15) / 16 * 16;   // float [2][64]; prologue scratch
  static constexpr int OFF_RED2 = OFF_RED + 2 * 4 * 16 * 4;    // float [2][4][8]: sums, zero-point terms
  static constexpr int OFF_QSC = OFF_RED2 + 2 * 4 * 8 * 4;     // float [8] scale, [8] sum(q)
  static constexpr int OFF_PMASK = OFF_QSC + 16 * 4;           // uint32 [NST] valid-page masks
  static constexpr int OFF_MISC = (OFF_PMASK + 4 * NST + 15) / 16 * 16;   // tmem base, abort flag, start (b, P)
  static constexpr int OFF_WALK = OFF_MISC + 32;               // softmax piece cursor [2] + slots [2][2]
  static constexpr int SMEM = OFF_WALK + 160 + 128;            // + alignment slack
  static_assert(OFF_RED % 16 == 0 && OFF_BAR % 8 == 0 && OFF_MISC % 16 == 0, "smem alignment");
};

// Context length of sequence b if it is legal, else 0.
__device__ __forceinline__ int mma_seq_ctx(const int32_t* ctx_lens, int b, int max_ctx, int W) {
  const int c = ctx_lens[b];
  return (c < 0 || c > max_ctx || int64_t(c) > int64_t(W) * kBlockSize) ? 0 : c;
}

// Work-list cost of one (sequence, KV head) run: its tiles plus kPieceCost
// virtual units in front of them, about what opening and closing a piece
// costs in tile times, so that equal shares of cost take equal time.
constexpr int kPieceCost = 1;

// Cursor over the pieces of one CTA's share [g, end) of the work list (cost
// units). Every role walks it the same way; the next sequence's length is
// loaded one sequence ahead so that stepping over a sequence boundary does not
// wait. A share that holds only a run's virtual units yields no piece there.
struct PieceWalk {
  int b, h, lo, hi;          // sequence, KV head, tiles [lo, hi) of that sequence
  int nt, ctx;               // tiles and tokens of sequence b
  int ctx_next;              // length of sequence b + 1 (0 past the batch)
  int gmask;                 // lengths are ANDed with it (~127: whole 128-token groups)
  long long P;               // cost per head of sequences 0 .. b-1
  long long g, gend, end;    // cost positions: this piece's start and end; end of the share
  bool done;

  __device__ __forceinline__ void load_next(const int32_t* ctx_lens, int B, int max_ctx, int W) {
    ctx_next = (b + 1 < B) ? (mma_seq_ctx(ctx_lens, b + 1, max_ctx, W) & gmask) : 0;
  }
  __device__ __forceinline__ void next_run(int Hk, const int32_t* ctx_lens, int B, int max_ctx,
                                           int W) {
    if (++h < Hk) return;
    h = 0;
    P += nt + kPieceCost;
    ++b;
    ctx = ctx_next;
    nt = (ctx + 127) / 128;
    load_next(ctx_lens, B, max_ctx, W);
    while (nt == 0) {                            // empty sequences hold no tiles
      ++b;
      ctx = ctx_next;
      nt = (ctx + 127) / 128;
      load_next(ctx_lens, B, max_ctx, W);
    }
  }
  // the piece starting at cost position g, or the next non-empty one
  __device__ __forceinline__ void settle(int Hk, const int32_t* ctx_lens, int B, int max_ctx,
                                         int W) {
    while (true) {
      if (g >= end) { done = true; return; }
      const long long L = nt + kPieceCost;
      const long long u = g - (int64_t(Hk) * P + int64_t(h) * L);   // offset in the run
      const long long uend = ll_min(L, u + (end - g));
      lo = int(ll_max(0, u - kPieceCost));
      hi = int(ll_max(0, uend - kPieceCost));
      gend = g + (uend - u);
      if (hi > lo) { done = false; return; }
      g = gend;
      if (g >= end) { done = true; return; }
      next_run(Hk, ctx_lens, B, max_ctx, W);
    }
  }
  __device__ __forceinline__ void init(int b0, long long P0, long long start, long long end_,
                                       int Hk, const int32_t* ctx_lens, int B, int max_ctx, int W,
                                       int gmask_ = -1) {
    b = b0; P = P0; g = start; end = end_;
    gmask = gmask_;
    ctx = mma_seq_ctx(ctx_lens, b, max_ctx, W) & gmask;
    nt = (ctx + 127) / 128;
    load_next(ctx_lens, B, max_ctx, W);
    lo = hi = 0;
    gend = g;
    if (g >= end || nt == 0) { done = true; h = 0; return; }
    h = int((g - int64_t(Hk) * P) / (nt + kPieceCost));
    settle(Hk, ctx_lens, B, max_ctx, W);
  }
  __device__ __forceinline__ void next(int Hk, const int32_t* ctx_lens, int B, int max_ctx, int W) {
    g = gend;
    if (g >= end) { done = true; return; }
    next_run(Hk, ctx_lens, B, max_ctx, W);
    settle(Hk, ctx_lens, B, max_ctx, W);
  }
  // cost position of tile 0 of run (b, h)
  __device__ __forceinline__ long long first_tile(int Hk) const {
    return int64_t(Hk) * P + int64_t(h) * (nt + kPieceCost) + kPieceCost;
  }
};

static_assert(2 * sizeof(PieceWalk) + 16 <= 160, "piece cursor area");

// Columns [0, N) (N a multiple of 8, at most 32) of this warp's TMEM lanes.
template <int N>
__device__ __forceinline__ void tmem_load_cols(uint32_t taddr, uint32_t* r) {
  static_assert(N % 8 == 0 && N <= 32, "columns");
  if constexpr (N >= 16) tc::tmem_ld16(taddr, *reinterpret_cast<uint32_t(*)[16]>(r));
  if constexpr (N == 32) tc::tmem_ld16(taddr + 16, *reinterpret_cast<uint32_t(*)[16]>(r + 16));
  if constexpr (N % 16 == 8) tc::tmem_ld8(taddr + (N - 8), r + (N - 8));
}

template <int D, int G, int FMT>
__global__ void __maxnreg__(FMT == KVQ_BF16 ? 168 : 120) decode_mma_kernel(
    const __nv_bfloat16* __restrict__ q, const uint8_t* __restrict__ kc,
    const uint8_t* __restrict__ vc, const __nv_bfloat16* __restrict__ ks,
    const __nv_bfloat16* __restrict__ vs, const int32_t* __restrict__ tables,
    const int32_t* __restrict__ ctx_lens, int B, int Hk, int nrg, int NB, int W, int max_ctx,
    int unit_tiles, int slots, float qk_scale, int per_tensor, int n_query,
    long long wait_limit, float* __restrict__ part_o,
    float* __restrict__ part_ml, int32_t* __restrict__ part_cnt) {
  using C = MmaCfg<D, G, FMT>;
  using namespace tc;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((128 - (smem_u32(smem_raw) & 127)) & 127);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int Hq = Hk * nrg * G;                             // query rows of a sequence
  // nrg CTAs form a group: they walk the same share of the (sequence, KV head,
  // tile) list in step, each for its own row group rg, so a page one of them
  // copies from HBM is in L2 for the others
  const int rg = int(blockIdx.x % nrg);
  const long long grp = blockIdx.x / nrg, NG = gridDim.x / nrg;

  uint8_t* kring = smem + C::OFF_K;
  uint8_t* vring = smem + C::OFF_V;
  uint8_t* kmeta = smem + C::OFF_KM;
  uint8_t* vmeta = smem + C::OFF_VM;
  uint8_t* qop = smem + C::OFF_Q;
  uint8_t* pop = smem + C::OFF_P;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* kfull = bars;
  uint64_t* kempty = bars + C::NST;
  uint64_t* vfull = bars + 2 * C::NST;
  uint64_t* vempty = bars + 3 * C::NST;
  uint64_t* sfull = bars + 4 * C::NST;      // [2]
  uint64_t* sfree = sfull + 2;              // [2]
  uint64_t* pready = sfree + 2;             // [2]
  uint64_t* ofull = pready + 2;             // [2]
  uint64_t* ofree = ofull + 2;              // [2]
  uint64_t* qready = ofree + 2;
  uint64_t* qfree = qready + 1;
  uint64_t* drain = qfree + 1;
  float* red = reinterpret_cast<float*>(smem + C::OFF_RED);
  float* red2 = reinterpret_cast<float*>(smem + C::OFF_RED2);
  float* qsc = reinterpret_cast<float*>(smem + C::OFF_QSC);
  float* qsum = qsc + 8;
  volatile uint32_t* pmask = reinterpret_cast<volatile uint32_t*>(smem + C::OFF_PMASK);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  // ------------------------------------------------------------ set-up
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NST; ++s) {
      mbar_init(kfull + s, 1);
      mbar_init(kempty + s, 128);
      mbar_init(vfull + s, 1);
      mbar_init(vempty + s, 1);
    }
    for (int j = 0; j < 2; ++j) {
      mbar_init(sfull + j, 1);
      mbar_init(sfree + j, 128);
      mbar_init(pready + j, 128);
      mbar_init(ofull + j, 1);
      mbar_init(ofree + j, 128);
    }
    mbar_init(qready, 128);
    mbar_init(qfree, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp >= 2) {
    // zero the query operand and both P buffers (padding rows stay zero)
    const int ct = threadIdx.x - 64;
    for (int i = ct * 16; i < C::QBYTES + 2 * C::PBYTES; i += 128 * 16)
      *reinterpret_cast<uint4*>(qop + i) = make_uint4(0, 0, 0, 0);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // Everything above (the barriers, the tensor memory) overlaps the kernel
  // ahead on the stream when this one is launched as its programmatic
  // dependent (the append of the same step) and touches no global memory: the
  // context lengths, query, block tables, scales and pages are read only after
  // that kernel has finished, whatever it wrote. The merge may launch now.
  grid_dep_wait();
  grid_dep_launch_dependents();

  // ------------------------------------------------------------ the share
  // T = total work-list cost; each thread sums the run costs of some sequences
  long long* red64 = reinterpret_cast<long long*>(smem + C::OFF_RED);   // [6] + 2
  long long* miscll = reinterpret_cast<long long*>(smem + C::OFF_MISC + 16);
  int* misci = reinterpret_cast<int*>(smem + C::OFF_MISC + 8);
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
  for (int w = 0; w < 6; ++w) T += red64[w];
  T *= Hk;
  const long long N = ll_min(NG, ll_max(1, T / max(1, unit_tiles)));
  if (T == 0 || grp >= N) {                               // uniform for the CTA
    if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
    return;
  }
  const long long start = (grp * T) / N;
  const long long end = ((grp + 1) * T) / N;
  // the sequence holding cost position `start`: block-wide scan of run costs
  {
    if (threadIdx.x == 0) misci[0] = -1;
    __syncthreads();
    long long run = 0;
    for (int base = 0; base < B; base += blockDim.x) {
      const int bb = base + threadIdx.x;
      int tb = bb < B ? (mma_seq_ctx(ctx_lens, bb, max_ctx, W) + 127) / 128 : 0;
      if (tb > 0) tb += kPieceCost;                           // run cost of sequence bb
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
      for (int w = 0; w < 6; ++w) {
        before += (w < warp) ? red64[w] : 0;
        total += red64[w];
      }
      const long long lo_t = run + before + incl - tb;          // run cost before sequence bb
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
  // group that holds work-list cost position x; the slot of a piece is its
  // group's rank among the groups that hold real tiles of the piece's (b, h)
  auto cta_of = [&](long long x) -> long long { return ((x + 1) * N - 1) / T; };

  PieceWalk walk;
  walk.init(b0, P0, start, end, Hk, ctx_lens, B, max_ctx, W);

  if (warp == 0) {
    // ---------------------------------------------------------- producer
    const uint64_t pol = l2_evict_first_policy();
    const int p8 = lane & 7;
    constexpr int CPP = C::METAB / 16;                    // 16-byte scale chunks per page
    // block id of page p8 of tile `tile` of the current piece of `pw`
    auto load_id = [&](const PieceWalk& pw, int tile) -> int {
      if (lane >= 8 || pw.done) return -2;
      const int tok0 = tile * 128;
      const int t1 = min(pw.hi * 128, pw.ctx);
      const int npg = min(8, (t1 - tok0 + kBlockSize - 1) / kBlockSize);
      return p8 < npg ? tables[int64_t(pw.b) * W + tok0 / kBlockSize + p8] : -2;   // -2: no page here
    };
    auto step = [&](PieceWalk& pw, int& tile) {
      if (pw.done) return;
      if (++tile >= pw.hi) {
        pw.next(Hk, ctx_lens, B, max_ctx, W);
        tile = pw.lo;
      }
    };
    // this lane's 16-byte chunk of the K and V scales of a tile (lane = page *
    // CPP + chunk), loaded one tile before it is stored into the stage
    const int sp = lane / (CPP > 0 ? CPP : 1), sc = lane % (CPP > 0 ? CPP : 1);
    auto load_scales = [&](int ids, int h, uint4& kv, uint4& vv) {
      kv = vv = make_uint4(0, 0, 0, 0);
      if constexpr (C::MV > 0) {
        const int sblk = __shfl_sync(0xffffffffu, ids, sp & 7);
        if (sp < 8 && sblk >= 0 && sblk < NB) {
          const int64_t off = (int64_t(sblk) * Hk + h) * C::METAB + sc * 16;
          kv = __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(ks) + off));
          vv = __ldg(reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(vs) + off));
        }
      }
    };
    // cursors of tiles gt, gt + 1, gt + 2; block ids are loaded two tiles ahead
    PieceWalk c0 = walk, c1 = walk, c2 = walk;
    int i0 = walk.lo, i1 = walk.lo, i2 = walk.lo;
    step(c1, i1);
    step(c2, i2);
    step(c2, i2);
    int id0 = load_id(c0, i0), id1 = load_id(c1, i1);
    uint4 ksc, vsc;
    load_scales(id0, c0.h, ksc, vsc);
    bool kiss[C::NST], viss[C::NST];
    uint32_t kpar[C::NST], vpar[C::NST];
#pragma unroll
    for (int s = 0; s < C::NST; ++s) { kiss[s] = viss[s] = false; kpar[s] = vpar[s] = 0; }
    for (int gt = 0; !c0.done; ++gt) {
      const int s = gt % C::NST;
      const uint32_t ph = (gt / C::NST) & 1;
      const int h = c0.h;
      const int id = id0;
      const int id2 = load_id(c2, i2);
      uint4 ksc_n, vsc_n;
      load_scales(c1.done ? -2 : id1, c1.h, ksc_n, vsc_n);   // next tile's scales, in flight
      if (lane < 8 && id != -2 && (id < 0 || id >= NB)) flag_error(KVQ_DEVERR_BLOCK);
      const bool valid = lane < 8 && id >= 0 && id < NB;
      const uint32_t mask = __ballot_sync(0xffffffffu, valid) & 0xFFu;
      const int blk = __shfl_sync(0xffffffffu, id, p8);
      const bool mine = ((mask >> p8) & 1u) != 0u;
      const bool smine = C::MV > 0 && sp < 8 && ((mask >> sp) & 1u) != 0u;
      const int64_t page = int64_t(blk) * Hk + h;
      const uint32_t bytes = uint32_t(__popc(mask)) * uint32_t(C::PAGE);
      bool ok = true;
      // per stage: byte count, the page copies, then the scale stores and the
      // one arrival that publishes them (the copies need not wait for the scales)
      if (lane == 0) {
        ok = mbar_wait(kempty + s, ph ^ 1, abort_flag, wait_limit);
        if (ok) mbar_expect_tx(kfull + s, bytes);
      }
      if (!__shfl_sync(0xffffffffu, int(ok), 0)) break;
      if (lane < 8 && mine) bulk_g2s(kring + (s * 8 + p8) * C::PAGE, kc + page * C::PAGE, C::PAGE, kfull + s, pol);
      kiss[s] = true;
      kpar[s] = ph;
      if (smine) *reinterpret_cast<uint4*>(kmeta + (s * 8 + sp) * C::METAB + sc * 16) = ksc;
      __syncwarp();
      if (lane == 0) {
        pmask[s] = mask;
        mbar_arrive(kfull + s);
      }
      if (lane == 0) {
        ok = mbar_wait(vempty + s, ph ^ 1, abort_flag, wait_limit);
        if (ok) mbar_expect_tx(vfull + s, bytes);
      }
      if (!__shfl_sync(0xffffffffu, int(ok), 0)) break;
      if (lane < 8 && mine) bulk_g2s(vring + (s * 8 + p8) * C::PAGE, vc + page * C::PAGE, C::PAGE, vfull + s, pol);
      viss[s] = true;
      vpar[s] = ph;
      if (smine) *reinterpret_cast<uint4*>(vmeta + (s * 8 + sp) * C::METAB + sc * 16) = vsc;
      __syncwarp();
      if (lane == 0) mbar_arrive(vfull + s);
      // shift the cursors
      c0 = c1; i0 = i1; id0 = id1; ksc = ksc_n; vsc = vsc_n;
      c1 = c2; i1 = i2; id1 = id2;
      step(c2, i2);
    }
    if (lane == 0 && *abort_flag) {
      // let the copies already issued land before the CTA's smem goes away
      volatile int no_abort = 0;
      for (int s = 0; s < C::NST; ++s) {
        if (kiss[s]) mbar_wait(kfull + s, kpar[s], &no_abort, kMmaWaitLimitCycles);
        if (viss[s]) mbar_wait(vfull + s, vpar[s], &no_abort, kMmaWaitLimitCycles);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t dfmt = C::I8 ? 2u : 1u;
      // A (cache codes): bf16 / s8 / E4M3 (0) or E5M2 (1); B (query and weight
      // parts): bf16 / s8 and u8 / E4M3, whatever FP8 variant the cache holds
      constexpr uint32_t afmt = (C::BF || C::I8 || FMT == KVQ_FP8_E5M2) ? 1u : 0u;
      constexpr uint32_t qfmt = (C::BF || C::I8) ? 1u : 0u;
      constexpr uint32_t pfmt = C::BF ? 1u : 0u;
      constexpr uint32_t id_s = idesc_m128(dfmt, afmt, qfmt, false, C::NS);
      constexpr uint32_t id_pv = idesc_m128(dfmt, afmt, pfmt, true, C::NO);
      const uint32_t kbase = smem_u32(kring), vbase = smem_u32(vring);
      const uint32_t qaddr = smem_u32(qop), paddr = smem_u32(pop);
      bool ok = true;
      int gt = 0;
      auto issue_pv = [&](int j) -> bool {
        const int s = j % C::NST;
        if (!mbar_wait(pready + (j & 1), (j >> 1) & 1, abort_flag, wait_limit)) return false;
        if (!mbar_wait(ofree + (j & 1), ((j >> 1) & 1) ^ 1, abort_flag, wait_limit)) return false;
        tc_fence_after();
        const uint32_t a0 = vbase + s * 8 * C::PAGE;
        const uint32_t b0 = paddr + (j & 1) * C::PBYTES;
#pragma unroll
        for (int kk = 0; kk < C::PV_MMAS; ++kk)
          mma_ss<C::KIND>(tmem + C::COL_O + (j & 1) * 32,
                          sdesc_plain(a0 + kk * 2 * C::V_LBO, C::V_LBO, C::V_SBO),
                          sdesc_plain(b0 + kk * (4 / C::E) * C::P_LBO, C::P_LBO, C::P_SBO), id_pv,
                          kk > 0);
        mma_commit(ofull + (j & 1));
        mma_commit(vempty + s);
        return true;
      };
      for (int pc = 0; ok && !walk.done; ++pc) {
        // the last tile of the piece before: its PV goes first, so that the
        // softmax warps can drain it while they build this piece's query
        if (gt >= 1) ok = issue_pv(gt - 1);
        // the query operand of piece pc (one buffer: the softmax warps rewrite
        // it only after every S product of the piece before has been read)
        if (ok) ok = mbar_wait(qready, pc & 1, abort_flag, wait_limit);
        tc_fence_after();
        const uint32_t qa = qaddr;
        for (int i = walk.lo; ok && i < walk.hi; ++i, ++gt) {
          const int s = gt % C::NST;
          ok = mbar_wait(kfull + s, (gt / C::NST) & 1, abort_flag, wait_limit) &&
               mbar_wait(sfree + (gt & 1), ((gt >> 1) & 1) ^ 1, abort_flag, wait_limit);
          if (!ok) break;
          tc_fence_after();
          const uint32_t a0 = kbase + s * 8 * C::PAGE;
#pragma unroll
          for (int kk = 0; kk < C::S_MMAS; ++kk)
            mma_ss<C::KIND>(tmem + C::COL_S + (gt & 1) * 32,
                            sdesc_plain(a0 + kk * 2 * C::K_LBO, C::K_LBO, C::K_SBO),
                            sdesc_plain(qa + kk * 2 * C::Q_LBO, C::Q_LBO, C::Q_SBO), id_s, kk > 0);
          mma_commit(sfull + (gt & 1));
          if (i > walk.lo) ok = issue_pv(gt - 1);
        }
        if (ok) mma_commit(qfree);                         // this piece's S products are issued
        walk.next(Hk, ctx_lens, B, max_ctx, W);
      }
      if (ok && gt >= 1) issue_pv(gt - 1);
      // every MMA issued so far completes before TMEM is released
      volatile int no_abort = 0;
      mma_commit(drain);
      mbar_wait(drain, 0, &no_abort, kMmaWaitLimitCycles);
    }
  } else {
    // ---------------------------------------------------------- softmax warps
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;                  // token / channel / TMEM lane
    const int cw = warp - 2;                            // query heads cw, cw + 4 of a piece
    const uint32_t lane_base = uint32_t(quarter * 32) << 16;
    bool ok = true;
    // this token's row of a P buffer (MN-major): element n at
    // (n / PT) * P_SBO + (n % PT) * E, plus the row's own offset
    const uint32_t prow = (r >> 3) * C::P_LBO + (r & 7) * 16;
    // The group's piece cursor lives in smem: wk[pc & 1] is piece pc, and
    // thread r == 0 advances it (with the piece's partial slot in pinfo) so
    // that no other thread keeps cursor state in registers.
    PieceWalk* wk = reinterpret_cast<PieceWalk*>(smem + C::OFF_WALK);
    int* pinfo = reinterpret_cast<int*>(smem + C::OFF_WALK + 2 * sizeof(PieceWalk));   // [2][2]
    auto publish = [&](int idx, const PieceWalk& pw) {
      wk[idx] = pw;
      if (!pw.done) {
        pinfo[idx * 2] = int(grp - cta_of(pw.first_tile(Hk)));
        pinfo[idx * 2 + 1] = pw.hi == pw.nt;
      }
    };
    if (r == 0) {
      publish(0, walk);
      PieceWalk n = walk;
      n.next(Hk, ctx_lens, B, max_ctx, W);
      publish(1, n);
    }
    named_bar_sync(1, 128);

    // query operand of a piece: the BF16 query rows of its group, loaded early
    // (qv) and written as exact parts later (store_q)
    float qv[C::HPW][D / 32];
    // static INT8: K scale of channel lane + 32 i of the piece's KV head; the
    // query is multiplied by it before the split, since sum_d q_d (s_d c_d) =
    // sum_d (q_d s_d) c_d
    [[maybe_unused]] float ksd[C::SI ? D / 32 : 1];
    auto load_q = [&](bool none, int qb, int qh) {
#pragma unroll
      for (int hh = 0; hh < C::HPW; ++hh) {
        const int g = cw + 4 * hh;
#pragma unroll
        for (int i = 0; i < D / 32; ++i)
          qv[hh][i] = (g < G && !none)
                          ? __bfloat162float(q[(int64_t(qb) * Hq + (qh * nrg + rg) * G + g) * D + lane + 32 * i])
                          : 0.f;
      }
      if constexpr (C::SI) {
#pragma unroll
        for (int i = 0; i < D / 32; ++i)
          ksd[i] = none ? 0.f : __bfloat162float(ks[per_tensor ? 0 : qh * D + lane + 32 * i]);
      }
    };
    // B operand of S (K-major, no swizzle): row n = part * G + g, element
    // (n, d) at (n/8)*Q_SBO + (n%8)*16 + (d*E/16)*Q_LBO + (d*E)%16
    auto store_q = [&]() {
#pragma unroll
      for (int hh = 0; hh < C::HPW; ++hh) {
        const int g = cw + 4 * hh;
        if (g >= G) continue;                                   // uniform per warp
        if constexpr (C::SI) {
#pragma unroll
          for (int i = 0; i < D / 32; ++i) qv[hh][i] *= ksd[i];
        }
        float amax = 0.f;
#pragma unroll
        for (int i = 0; i < D / 32; ++i) amax = fmaxf(amax, fabsf(qv[hh][i]));
        amax = warp_max(amax);
        // power-of-two scaling of the head: FP8 puts max|q| into [128, 256)
        // (inside the E4M3 range), INT8 into [32, 64) (parts within +-64)
        int e = 0;
        if (!C::BF && amax > 0.f) e = (C::F8 ? 7 : 5) - ilogbf(amax);
        e = max(-120, min(120, e));
        const float up = __int_as_float((127 + e) << 23);
        const float down = __int_as_float((127 - e) << 23);
        int isum = 0;
#pragma unroll
        for (int i = 0; i < D / 32; ++i) {
          const int d = lane + 32 * i;
          auto at = [&](int n) -> uint8_t* {
            return qop + (n >> 3) * C::Q_SBO + (n & 7) * 16 + ((d * C::E) >> 4) * C::Q_LBO +
                   ((d * C::E) & 15);
          };
          if constexpr (C::BF) {
            *reinterpret_cast<uint16_t*>(at(g)) = __bfloat16_as_ushort(__float2bfloat16_rn(qv[hh][i]));
          } else if constexpr (C::F8) {
            // x = hi + lo/16 with both parts E4M3: exact for a BF16 value unless
            // it lies below the E4M3 normal range after scaling
            const float x = qv[hh][i] * up;
            const uint32_t hc = f32x2_to_e4m3x2(x, 0.f) & 0xFFu;
            float hv, unused;
            e4m3x2_to_f32x2(hc, hv, unused);
            const uint32_t lc = f32x2_to_e4m3x2((x - hv) * 16.f, 0.f) & 0xFFu;
            *at(g) = uint8_t(hc);
            *at(G + g) = uint8_t(lc);
          } else {
            // x = x0 + x1/128 + x2/16384, every part an integer in [-64, 64]
            const float x = qv[hh][i] * up;
            const float x0 = rintf(x);
            const float r0 = (x - x0) * 128.f;
            const float x1 = rintf(r0);
            const float x2 = rintf((r0 - x1) * 128.f);
            const int i0 = int(x0), i1 = int(x1), i2 = int(x2);
            *at(g) = uint8_t(int8_t(i0));
            *at(G + g) = uint8_t(int8_t(i1));
            *at(2 * G + g) = uint8_t(int8_t(i2));
            isum += i0 * 16384 + i1 * 128 + i2;
          }
        }
        if constexpr (C::ZP) {
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) isum += __shfl_xor_sync(0xffffffffu, isum, o);
        }
        if (lane == 0) {
          qsc[g] = qk_scale * down;
          qsum[g] = float(isum) * (1.f / 16384.f);             // sum of q in the units of S
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
    };

    // first piece's query operand
    load_q(wk[0].done, wk[0].b, wk[0].h);
    store_q();
    mbar_arrive(qready);

    int gt = 0;
    for (int pc = 0;; ++pc) {
      const PieceWalk* cur = wk + (pc & 1);
      const PieceWalk* nxt = wk + ((pc + 1) & 1);
      if (cur->done) break;                              // uniform
      const int pb = cur->b, ph_ = cur->h, lo = cur->lo, hi = cur->hi;
      const int t1 = min(hi * 128, cur->ctx);
      const int pctx = cur->ctx;
      const int slot = pinfo[(pc & 1) * 2], last = pinfo[(pc & 1) * 2 + 1];
      const bool more = !nxt->done;
      load_q(!more, nxt->b, nxt->h);                     // next piece's query, in flight
      named_bar_sync(1, 128);                            // all read the cursor; qsc/qsum visible
      if (r == 0) {                                      // piece pc + 2 into this piece's entry
        PieceWalk n = *nxt;
        if (!n.done) n.next(Hk, ctx_lens, B, max_ctx, W);
        publish(pc & 1, n);
      }
      float qs[G], qz[G];
#pragma unroll
      for (int g = 0; g < G; ++g) { qs[g] = qsc[g]; qz[g] = qsum[g]; }
      float m[G], l[G], corr[G], o[G], alpha[G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        m[g] = -INFINITY; l[g] = 0.f; corr[g] = 0.f; o[g] = 0.f; alpha[g] = 1.f;
      }
      float einv_pend = 1.f;

      // o (relative to the current max) += O tile j * 2^-e_j * alpha: alpha
      // moves tile j from the max it was weighted with to the current one
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
          float v;
          if constexpr (C::F8) {
            v = __uint_as_float(ov[g]) + __uint_as_float(ov[G + g]) * 0.0625f +
                __uint_as_float(ov[2 * G + g]) * (1.f / 256.f) +
                __uint_as_float(ov[3 * G + g]) * (1.f / 4096.f);
          } else if constexpr (C::I8) {
            v = float(int(ov[g])) + float(int(ov[G + g])) * (1.f / 256.f) +
                float(int(ov[2 * G + g])) * (1.f / 65536.f);
          } else {
            v = __uint_as_float(ov[g]) + __uint_as_float(ov[G + g]) + __uint_as_float(ov[2 * G + g]);
          }
          o[g] += v * (einv_pend * alpha[g]);
        }
      };

      for (int i = lo; i < hi; ++i, ++gt) {
        const int s = gt % C::NST;
        // ---- S of tile gt
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

        // ---- this token's scales (both copies acquired here, not through the MMA)
        if (ok) ok = mbar_wait(kfull + s, (gt / C::NST) & 1, abort_flag, wait_limit);
        if (ok) ok = mbar_wait(vfull + s, (gt / C::NST) & 1, abort_flag, wait_limit);
        const uint32_t mask = ok ? pmask[s] : 0u;   // pages of the tile with legal ids
        const int tile0 = i * 128;
        const int p = r >> 4, t = r & 15;
        const bool valid = ok && ((mask >> p) & 1u) && (tile0 + r < t1);
        float sk = 1.f, zk = 0.f, sv = 0.f, zv = 0.f;
        if (valid) {
          if constexpr (C::F8) {
            sk = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(kmeta + (s * 8 + p) * C::METAB)[t]);
            sv = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(vmeta + (s * 8 + p) * C::METAB)[t]);
          } else if constexpr (C::ZP) {
            const __nv_bfloat162 km = reinterpret_cast<const __nv_bfloat162*>(kmeta + (s * 8 + p) * C::METAB)[t];
            const __nv_bfloat162 vm = reinterpret_cast<const __nv_bfloat162*>(vmeta + (s * 8 + p) * C::METAB)[t];
            sk = __low2float(km); zk = __high2float(km);
            sv = __low2float(vm); zv = __high2float(vm);
          } else {
            sv = 1.f;                            // BF16 and static INT8: no per-token scales
          }
        }
        mbar_arrive(kempty + s);

        // ---- scores (base 2) and the tile max of every head
        float x[G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
          float sc;
          if constexpr (C::F8) {
            sc = __uint_as_float(sw[g]) + __uint_as_float(sw[G + g]) * 0.0625f;
          } else if constexpr (C::I8) {
            sc = float(int(sw[g])) + float(int(sw[G + g])) * (1.f / 128.f) +
                 float(int(sw[2 * G + g])) * (1.f / 16384.f);
            if constexpr (C::ZP) sc -= zk * qz[g];
          } else {
            sc = __uint_as_float(sw[g]);
          }
          x[g] = valid ? sc * sk * qs[g] : -INFINITY;
        }
        if (n_query > 1) {
          // multi-query: row rr = rg * G + g of the KV head's rows is query
          // position j = rr % n_query of query head rr / n_query,
          // and position j sees the tokens before the last n_query - 1 - j of
          // the context
          const int after = pctx - 1 - (tile0 + r);       // tokens after this one
          const int rr0 = rg * G;
#pragma unroll
          for (int g = 0; g < G; ++g)
            if (n_query - 1 - (rr0 + g) % n_query > after) x[g] = -INFINITY;
        }
        // per-head tile maxima of the four warps, head-major: rb[g][quarter]
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
        // P = p * v_scale * 2^ex with max(v_scale) * 2^ex in [128, 256): inside
        // the E4M3 range, and below 2^8 for the 24-bit fixed point of INT8
        const float4 s4 = *reinterpret_cast<const float4*>(rb + 8 * 4);
        const float svmax = fmaxf(fmaxf(s4.x, s4.y), fmaxf(s4.z, s4.w));
        int ex = 0;
        if (!C::BF && svmax > 0.f) ex = max(-120, min(120, 7 - ilogbf(svmax)));
        const float escale = __int_as_float((127 + ex) << 23);
        const float einv = __int_as_float((127 - ex) << 23);

        // ---- tokens of this tile past the sequence end or on a missing page:
        // their V rows in smem are stale or never written; zero them so that
        // 0 * (stale code) cannot produce a NaN (integer codes need no care)
        if constexpr (!C::I8) {
          if (mask != 0xFFu || tile0 + 128 > t1) {          // uniform over the CTA
            if (r < D) {
#pragma unroll 1
              for (int pp = 0; pp < 8; ++pp) {
                int ntok = ((mask >> pp) & 1u) ? t1 - (tile0 + 16 * pp) : 0;
                ntok = max(0, min(16, ntok));
                if (ntok == 16) continue;
                uint8_t* vpg = vring + (s * 8 + pp) * C::PAGE;
#pragma unroll
                for (int u = 0; u < C::E; ++u) {                 // 16-byte chunks of row r
                  uint4* cp = reinterpret_cast<uint4*>(vpg + u * (D * 16) + r * 16);
                  uint4 w = *cp;
                  uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                  for (int e = 0; e < 4; ++e) {
                    uint32_t keep = 0;
#pragma unroll
                    for (int bb = 0; bb < 4; ++bb) {
                      const int tok = (u * 16 + e * 4 + bb) / C::E;   // token of byte bb of word e
                      if (tok < ntok) keep |= 0xFFu << (8 * bb);
                    }
                    ww[e] &= keep;
                  }
                  *cp = make_uint4(ww[0], ww[1], ww[2], ww[3]);
                }
              }
            }
          }
        }

        // ---- weights -> P buffer (gt & 1), the row of token r
        uint8_t* pbuf = pop + (gt & 1) * C::PBYTES + prow;
        if constexpr (C::F8) {
          // y = y0 + y1/16 + y2/256 + y3/4096, each part E4M3 (RNE); the
          // residual is exact in FP32 and 16x smaller than the part before
          float y[G];
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const float pr = x[g] != -INFINITY ? exp2f(x[g] - m[g]) : 0.f;
            l[g] = l[g] * alpha[g] + pr;
            y[g] = pr * sv * escale;
          }
          uint32_t words[C::NO / 4];
#pragma unroll
          for (int e = 0; e < C::NO / 4; ++e) words[e] = 0u;
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) {
#pragma unroll
            for (int g = 0; g < G; g += 2) {
              const float a = y[g];
              const float c = (g + 1 < G) ? y[g + 1] : 0.f;
              const uint32_t code2 = f32x2_to_e4m3x2(a, c);
              const int n = jj * G + g;                        // byte index in the row
              words[n >> 2] |= code2 << (8 * (n & 3));
              if (jj < 3) {
                float av, cv;
                e4m3x2_to_f32x2(code2, av, cv);
                y[g] = (a - av) * 16.f;
                if (g + 1 < G) y[g + 1] = (c - cv) * 16.f;
              }
            }
          }
#pragma unroll
          for (int c16 = 0; c16 < C::NO / 16; ++c16)
            *reinterpret_cast<uint4*>(pbuf + c16 * C::P_SBO) =
                make_uint4(words[4 * c16], words[4 * c16 + 1], words[4 * c16 + 2], words[4 * c16 + 3]);
        } else if constexpr (C::I8) {
          // Y = rint(y * 2^16) < 2^24; its three bytes are the parts (weights
          // 1, 1/256, 1/65536); zero_point * P is summed from the same Y
          uint32_t yv[G];
          const float ysc = sv * escale * 65536.f;
          [[maybe_unused]] const float zsc = zv * einv * (1.f / 65536.f);
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const float pr = x[g] != -INFINITY ? exp2f(x[g] - m[g]) : 0.f;
            l[g] = l[g] * alpha[g] + pr;
            yv[g] = __float2uint_rn(pr * ysc);
            if constexpr (C::ZP) corr[g] = corr[g] * alpha[g] + float(yv[g]) * zsc;
          }
          uint32_t words[C::NO / 4];
#pragma unroll
          for (int e = 0; e < C::NO / 4; ++e) words[e] = 0u;
          if constexpr (G % 4 == 0) {
            // byte b = 2 - jj of four heads' Y into one word: three byte permutes
#pragma unroll
            for (int jj = 0; jj < 3; ++jj) {
              const uint32_t sel = uint32_t(2 - jj) | (uint32_t(6 - jj) << 4);
#pragma unroll
              for (int g = 0; g < G; g += 4) {
                const uint32_t lo = __byte_perm(yv[g], yv[g + 1], sel);
                const uint32_t hi = __byte_perm(yv[g + 2], yv[g + 3], sel);
                words[(jj * G + g) >> 2] = __byte_perm(lo, hi, 0x5410);
              }
            }
          } else {
#pragma unroll
            for (int jj = 0; jj < 3; ++jj) {
#pragma unroll
              for (int g = 0; g < G; ++g) {
                const int n = jj * G + g;
                words[n >> 2] |= ((yv[g] >> (16 - 8 * jj)) & 0xFFu) << (8 * (n & 3));
              }
            }
          }
#pragma unroll
          for (int c16 = 0; c16 < C::NO / 16; ++c16)
            *reinterpret_cast<uint4*>(pbuf + c16 * C::P_SBO) =
                make_uint4(words[4 * c16], words[4 * c16 + 1], words[4 * c16 + 2], words[4 * c16 + 3]);
        } else {
          // p = hi + mid + lo, each bf16: 24 significant bits
          uint32_t words[C::NO / 2];
#pragma unroll
          for (int e = 0; e < C::NO / 2; ++e) words[e] = 0u;
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const float pr = x[g] != -INFINITY ? exp2f(x[g] - m[g]) : 0.f;
            l[g] = l[g] * alpha[g] + pr;
            const __nv_bfloat16 hi = __float2bfloat16_rn(pr);
            const float r1 = pr - __bfloat162float(hi);
            const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
            const __nv_bfloat16 lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
            const uint16_t parts[3] = {__bfloat16_as_ushort(hi), __bfloat16_as_ushort(mid),
                                       __bfloat16_as_ushort(lo)};
#pragma unroll
            for (int jj = 0; jj < 3; ++jj) {
              const int n = jj * G + g;
              words[n >> 1] |= uint32_t(parts[jj]) << (16 * (n & 1));
            }
          }
#pragma unroll
          for (int c8 = 0; c8 < C::NO / 8; ++c8)
            *reinterpret_cast<uint4*>(pbuf + c8 * C::P_SBO) =
                make_uint4(words[4 * c8], words[4 * c8 + 1], words[4 * c8 + 2], words[4 * c8 + 3]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(pready + (gt & 1));

        // ---- O of the previous tile of this piece
        if (i > lo) accum_o(gt - 1);
        einv_pend = einv;
      }

      // ---- the next piece's query operand, so that its first S can start
      // while this piece's last O drains
      if (more) {
        if (ok) ok = mbar_wait(qfree, pc & 1, abort_flag, wait_limit);
        store_q();
        mbar_arrive(qready);
      }
#pragma unroll
      for (int g = 0; g < G; ++g) alpha[g] = 1.f;
      accum_o(gt - 1);

      // ---- piece partial: (max, sum, unnormalised output) per query head
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float ls = warp_sum(l[g]);
        const float cs = C::ZP ? warp_sum(corr[g]) : 0.f;
        if (lane == 0) {
          red2[quarter * 8 + g] = ls;
          red2[32 + quarter * 8 + g] = cs;
        }
      }
      named_bar_sync(1, 128);
      // static INT8: the V scale of channel r multiplies the finished sums
      float vsd = 1.f;
      if constexpr (C::SI) {
        if (r < D) vsd = __bfloat162float(vs[per_tensor ? 0 : ph_ * D + r]);
      }
      // After a wait ran out the piece's sums are incomplete: it writes a
      // marker instead (max +inf, sum and output NaN), so that every output row
      // the piece contributes to merges to NaN rather than to a plausible value
      // built from stale workspace.
      const bool good = ok && !*abort_flag;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float L = red2[g] + red2[8 + g] + red2[16 + g] + red2[24 + g];
        const float Cz = red2[32 + g] + red2[40 + g] + red2[48 + g] + red2[56 + g];
        const int64_t row = (int64_t(pb) * Hq + (ph_ * nrg + rg) * G + g) * slots + slot;
        if (r < D) part_o[row * D + r] = good ? (o[g] - Cz) * vsd : __int_as_float(0x7fc00000);
        if (r == 0) {
          part_ml[row * 2] = good ? m[g] : INFINITY;
          part_ml[row * 2 + 1] = good ? L : __int_as_float(0x7fc00000);
        }
      }
      if (r == 0 && last) part_cnt[(int64_t(pb) * Hk + ph_) * nrg + rg] = slot + 1;
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

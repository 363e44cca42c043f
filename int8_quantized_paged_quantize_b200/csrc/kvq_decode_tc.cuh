// Paged GQA decode attention on the 5th-generation tensor cores (tcgen05, TMEM).
// Included by kvq_kernels.cu (it shares the device error word).
//
// One CTA per (sequence b, KV head h, chunk of `part` tokens), 6 warps:
//   warp 0      producer: for each 128-token tile (8 pages of 16 tokens) it
//               walks the block table and issues 1-D bulk copies (TMA engine)
//               of the K pages, V pages and their scales into a ring of smem
//               stages, completed on mbarriers with byte counts;
//   warp 1      allocates TMEM and issues the MMAs from one thread;
//   warps 2..5  compute warps, one per TMEM lane quarter; thread r of the
//               group owns token r of the tile (K, softmax) and channel r (V, O).
// Per tile:
//   K codes -> exact f16 values (E4M3 via cvt, INT8 as c - zp, BF16 as is) ->
//     TMEM: A of S^T[128 tok x 16] = K[128 x D] . Q^T[D x 16] (Q^T in smem,
//     128-byte swizzle, the GQA group in the first G rows).
//   softmax (base 2) per token row in FP32 registers; the tile max of every
//     head is exchanged through smem; the weight p * s_v (V scale folded in)
//     is scaled by a per-tile power of two and split into two f16 parts
//     (hi + lo carry 22 significant bits) -> smem, B of the PV product.
//   V codes -> exact f16 values -> TMEM: A of O^T[D x (2 x 8)] = V^T . P.
//   O tile -> registers, rescaled and accumulated in FP32.
// The same scheme runs the BF16 cache with bf16 operands and P split in three
// bf16 parts. Every byte of the chunk's K/V is read from HBM once for the whole
// query group. Every wait is bounded: on expiry the CTA sets KVQ_DEVERR_TIMEOUT,
// stops issuing work, drains what it issued, frees TMEM and returns.

#pragma once

#include "kvq_tc.cuh"

namespace kvq {

constexpr long long kWaitLimitCycles = 2000000000LL;   // about one second

template <int D, int FMT>
struct TcCfg {
  static constexpr bool BF = FMT == KVQ_BF16;
  static constexpr int ELT = BF ? 2 : 1;
  static constexpr int PAGE = kBlockSize * D * ELT;          // bytes of one (block, head) page
  static constexpr int NST = BF ? 2 : 3;                     // smem ring stages
  static constexpr int MV = FMT == KVQ_FP8_E4M3 ? 1 : (FMT == KVQ_INT8_ASYM ? 2 : 0);
  static constexpr int METAB = kBlockSize * MV * 2;          // scale bytes per page
  static constexpr int KCH = D * ELT / 16;                   // 16-byte chunks per K row
  static constexpr int KWORDS = D / 2;                       // 32-bit TMEM columns per K row
  static constexpr int NPARTS = BF ? 3 : 2;                  // parts of the split weight
  static constexpr int NPR = BF ? 32 : 16;                   // rows of the P operand (PV N)
  static constexpr int KSTEPS_QK = D / 16;
  // TMEM columns
  static constexpr int COL_AK0 = 0, COL_AK1 = 64, COL_AV = 128;
  static constexpr int COL_S0 = 192, COL_S1 = 208, COL_O0 = 224, COL_O1 = 224 + NPR;
  static constexpr int TMEM_COLS = BF ? 512 : 256;
  // shared memory carve-up (offsets from a 1024-aligned base)
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + NST * 8 * PAGE;
  static constexpr int OFF_KM = OFF_V + NST * 8 * PAGE;
  static constexpr int OFF_VM = OFF_KM + NST * 8 * METAB;
  static constexpr int OFF_Q = ((OFF_VM + NST * 8 * METAB) + 1023) / 1024 * 1024;
  static constexpr int QATOM = 16 * 128;                     // 16 rows x 64 values
  static constexpr int QBYTES = QATOM * (D / 64);
  static constexpr int OFF_P = OFF_Q + QBYTES;
  static constexpr int PATOM = NPR * 128;
  static constexpr int PBYTES = 2 * PATOM;                   // 128 tokens = 2 atoms
  static constexpr int OFF_BAR = OFF_P + 2 * PBYTES;
  static constexpr int NBAR = 4 * NST + 8;
  static constexpr int OFF_RED = OFF_BAR + 8 * NBAR;         // float [2][4][16]
  static constexpr int OFF_RED2 = OFF_RED + 2 * 4 * 16 * 4;  // float [2][4][8]
  static constexpr int OFF_QSC = OFF_RED2 + 2 * 4 * 8 * 4;   // float [8]
  static constexpr int OFF_PMASK = OFF_QSC + 8 * 4;          // uint32 [NST] valid-page masks
  static constexpr int OFF_MISC = OFF_PMASK + 4 * NST;       // tmem base, abort flag
  static constexpr int SMEM = OFF_MISC + 16 + 1024;          // + alignment slack
};

template <int D, int G, int FMT>
__global__ void __launch_bounds__(192, FMT == KVQ_BF16 ? 1 : 2) decode_tc_kernel(
    const __nv_bfloat16* __restrict__ q, const uint8_t* __restrict__ kc,
    const uint8_t* __restrict__ vc, const __nv_bfloat16* __restrict__ ks,
    const __nv_bfloat16* __restrict__ vs, const int32_t* __restrict__ tables,
    const int32_t* __restrict__ ctx_lens, int Hk, int NB, int W, int max_ctx, int part,
    int max_splits, float qk_scale, float* __restrict__ part_o, float* __restrict__ part_ml,
    int slots, int32_t* __restrict__ part_cnt) {
  using C = TcCfg<D, FMT>;
  using namespace tc;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x % max_splits;
  const int bh = blockIdx.x / max_splits;
  const int b = bh / Hk, h = bh % Hk;
  const int Hq = Hk * G;

  int ctx = ctx_lens[b];
  if (ctx < 0 || ctx > max_ctx || int64_t(ctx) > int64_t(W) * kBlockSize) {
    if (threadIdx.x == 0 && split == 0) flag_error(KVQ_DEVERR_CONTEXT);
    ctx = 0;
  }
  const int n_splits = (ctx + part - 1) / part;
  if (split >= n_splits) return;                         // uniform for the CTA
  const int t0 = split * part, t1 = min(ctx, t0 + part);
  const int ntiles = (t1 - t0 + 127) / 128;
  const int32_t* trow = tables + int64_t(b) * W;

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
  uint64_t* akfull = bars + 4 * C::NST;     // [2]
  uint64_t* sfull = akfull + 2;             // [2]
  uint64_t* ofull = sfull + 2;              // [2]
  uint64_t* pvready = ofull + 2;
  uint64_t* drain = pvready + 1;
  float* red = reinterpret_cast<float*>(smem + C::OFF_RED);
  float* red2 = reinterpret_cast<float*>(smem + C::OFF_RED2);
  float* qsc = reinterpret_cast<float*>(smem + C::OFF_QSC);
  volatile uint32_t* pmask = reinterpret_cast<volatile uint32_t*>(smem + C::OFF_PMASK);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  // ------------------------------------------------------------ set-up
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NST; ++s) {
      mbar_init(kfull + s, 1);
      mbar_init(kempty + s, 128);
      mbar_init(vfull + s, 1);
      mbar_init(vempty + s, 128);
    }
    for (int j = 0; j < 2; ++j) {
      mbar_init(akfull + j, 128);
      mbar_init(sfull + j, 1);
      mbar_init(ofull + j, 1);
    }
    mbar_init(pvready, 128);
    mbar_init(drain, 1);
    *abort_flag = 0;
    mbar_init_fence();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp >= 2) {
    const int ct = threadIdx.x - 64;                       // 0..127
    // zero the Q and P operands (padding rows stay zero)
    for (int i = ct * 16; i < C::QBYTES + 2 * C::PBYTES; i += 128 * 16)
      *reinterpret_cast<uint4*>(qop + i) = make_uint4(0, 0, 0, 0);
    named_bar_sync(1, 128);
    // Q^T of the group: row g = query head h*G + g. For the 8-bit caches the
    // BF16 query is scaled by an exact power of two (largest |q| into
    // [2^14, 2^15)) and stored as f16; the scale is undone in qsc[g].
    const int cw = warp - 2;
    for (int g = cw; g < G; g += 4) {
      const __nv_bfloat16* qr = q + (int64_t(b) * Hq + h * G + g) * D;
      float v[D / 32];
      float amax = 0.f;
#pragma unroll
      for (int i = 0; i < D / 32; ++i) {
        v[i] = __bfloat162float(qr[lane + 32 * i]);
        amax = fmaxf(amax, fabsf(v[i]));
      }
      amax = warp_max(amax);
      int e = 0;
      if (!C::BF && amax > 0.f) e = 14 - ilogbf(amax);
      e = max(-120, min(120, e));
      const float up = C::BF ? 1.f : __int_as_float((127 + e) << 23);
      const float down = C::BF ? 1.f : __int_as_float((127 - e) << 23);
#pragma unroll
      for (int i = 0; i < D / 32; ++i) {
        const int d = lane + 32 * i;
        uint16_t bits;
        if constexpr (C::BF) bits = __bfloat16_as_ushort(__float2bfloat16_rn(v[i]));
        else bits = __half_as_ushort(__float2half_rn(v[i] * up));
        *reinterpret_cast<uint16_t*>(qop + sw128_offset(g, d, 16)) = bits;
      }
      if (lane == 0) qsc[g] = qk_scale * down;
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      const uint64_t pol = l2_evict_first_policy();
      int last_parity[C::NST];
      bool issued[C::NST];
#pragma unroll
      for (int s = 0; s < C::NST; ++s) { issued[s] = false; last_parity[s] = 0; }
      for (int i = 0; i < ntiles; ++i) {
        const int s = i % C::NST;
        const uint32_t ph = (i / C::NST) & 1;
        const int tok0 = t0 + 128 * i;
        const int pg0 = tok0 / kBlockSize;
        const int npg = min(8, (t1 - tok0 + kBlockSize - 1) / kBlockSize);
        int blk[8];
        uint32_t nvalid = 0;
#pragma unroll
        for (int p = 0; p < 8; ++p) {
          blk[p] = p < npg ? trow[pg0 + p] : -1;
          if (p < npg && (blk[p] < 0 || blk[p] >= NB)) {
            flag_error(KVQ_DEVERR_BLOCK);
            blk[p] = -1;
          }
          nvalid += blk[p] >= 0;
        }
        uint32_t mask = 0;
#pragma unroll
        for (int p = 0; p < 8; ++p) mask |= (blk[p] >= 0 ? 1u : 0u) << p;
        if (!mbar_wait(kempty + s, ph ^ 1, abort_flag, kWaitLimitCycles)) break;
        pmask[s] = mask;                       // published by the arrive below
        mbar_arrive_expect_tx(kfull + s, nvalid * uint32_t(C::PAGE + C::METAB));
#pragma unroll
        for (int p = 0; p < 8; ++p) {
          if (blk[p] < 0) continue;
          const int64_t page = int64_t(blk[p]) * Hk + h;
          bulk_g2s(kring + (s * 8 + p) * C::PAGE, kc + page * C::PAGE, C::PAGE, kfull + s, pol);
          if constexpr (C::MV > 0)
            bulk_g2s(kmeta + (s * 8 + p) * C::METAB,
                     reinterpret_cast<const uint8_t*>(ks) + page * C::METAB, C::METAB, kfull + s, pol);
        }
        if (!mbar_wait(vempty + s, ph ^ 1, abort_flag, kWaitLimitCycles)) {
          issued[s] = true;
          last_parity[s] = ph;
          break;
        }
        mbar_arrive_expect_tx(vfull + s, nvalid * uint32_t(C::PAGE + C::METAB));
#pragma unroll
        for (int p = 0; p < 8; ++p) {
          if (blk[p] < 0) continue;
          const int64_t page = int64_t(blk[p]) * Hk + h;
          bulk_g2s(vring + (s * 8 + p) * C::PAGE, vc + page * C::PAGE, C::PAGE, vfull + s, pol);
          if constexpr (C::MV > 0)
            bulk_g2s(vmeta + (s * 8 + p) * C::METAB,
                     reinterpret_cast<const uint8_t*>(vs) + page * C::METAB, C::METAB, vfull + s, pol);
        }
        issued[s] = true;
        last_parity[s] = ph;
      }
      if (*abort_flag) {
        // let the copies already issued land before the CTA's smem goes away
        volatile int no_abort = 0;
        for (int s = 0; s < C::NST; ++s)
          if (issued[s]) {
            mbar_wait(kfull + s, last_parity[s], &no_abort, kWaitLimitCycles);
            mbar_wait(vfull + s, last_parity[s], &no_abort, kWaitLimitCycles);
          }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idq = idesc_f16(16, C::BF);
      constexpr uint32_t idp = idesc_f16(C::NPR, C::BF);
      const uint32_t qaddr = smem_u32(qop), paddr = smem_u32(pop);
      auto issue_s = [&](int j) -> bool {
        if (!mbar_wait(akfull + (j & 1), (j >> 1) & 1, abort_flag, kWaitLimitCycles)) return false;
        tc_fence_after();
        const uint32_t dt = tmem + ((j & 1) ? C::COL_S1 : C::COL_S0);
        const uint32_t at = tmem + ((j & 1) ? C::COL_AK1 : C::COL_AK0);
#pragma unroll
        for (int kk = 0; kk < C::KSTEPS_QK; ++kk)
          mma_f16_ts(dt, at + 8 * kk, sdesc_sw128(qaddr + (kk >> 2) * C::QATOM + (kk & 3) * 32), idq,
                     kk > 0);
        mma_commit(sfull + (j & 1));
        return true;
      };
      auto issue_pv = [&](int i) -> bool {
        if (!mbar_wait(pvready, i & 1, abort_flag, kWaitLimitCycles)) return false;
        tc_fence_after();
        const uint32_t dt = tmem + ((i & 1) ? C::COL_O1 : C::COL_O0);
        const uint32_t pb = paddr + (i & 1) * C::PBYTES;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_f16_ts(dt, tmem + C::COL_AV + 8 * kk,
                     sdesc_sw128(pb + (kk >> 2) * C::PATOM + (kk & 3) * 32), idp, kk > 0);
        mma_commit(ofull + (i & 1));
        return true;
      };
      bool ok = issue_s(0);
      for (int i = 0; ok && i < ntiles; ++i) {
        if (i + 1 < ntiles) ok = issue_s(i + 1);
        if (ok) ok = issue_pv(i);
      }
      // every MMA issued so far completes before TMEM is released
      volatile int no_abort = 0;
      mma_commit(drain);
      mbar_wait(drain, 0, &no_abort, kWaitLimitCycles);
    }
  } else {
    // ---------------------------------------------------------- compute warps
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;                  // token / channel / TMEM lane
    const uint32_t lane_base = uint32_t(quarter * 32) << 16;
    float qs[G];
#pragma unroll
    for (int g = 0; g < G; ++g) qs[g] = qsc[g];
    float m[G], l[G], corr[G], o[G], alpha_pend[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      m[g] = -INFINITY; l[g] = 0.f; corr[g] = 0.f; o[g] = 0.f; alpha_pend[g] = 1.f;
    }
    float einv_pend = 1.f;
    bool ok = true;
    // byte offset of (row g, token r) in a P buffer; row part*8 + g adds part*1024
    uint32_t poff[G];
#pragma unroll
    for (int g = 0; g < G; ++g) poff[g] = sw128_offset(g, r, C::NPR);
    // carried from the K conversion of tile j to the softmax/V of tile j
    float sk_carry = 0.f, sk_cur = 0.f;
    uint32_t valid_carry = 0, valid_cur = 0;

    auto conv_k = [&](int j) {
      const int s = j % C::NST;
      if (ok) ok = mbar_wait(kfull + s, (j / C::NST) & 1, abort_flag, kWaitLimitCycles);
      const uint32_t mask = ok ? pmask[s] : 0u;   // pages of tile j inside the chunk with legal ids
      const int p = r >> 4, t = r & 15;
      const bool valid = ok && (mask >> p & 1) && (t0 + 128 * j + r < t1);
      uint32_t w[C::KWORDS];
      float sk = 0.f;
      if (valid) {
        const uint8_t* pg = kring + (s * 8 + p) * C::PAGE;
        float zk = 0.f;
        if constexpr (FMT == KVQ_FP8_E4M3) {
          sk = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(kmeta + (s * 8 + p) * C::METAB)[t]);
        } else if constexpr (FMT == KVQ_INT8_ASYM) {
          const __nv_bfloat16* mm = reinterpret_cast<const __nv_bfloat16*>(kmeta + (s * 8 + p) * C::METAB);
          sk = __bfloat162float(mm[2 * t]);
          zk = __bfloat162float(mm[2 * t + 1]);
        } else {
          sk = 1.f;
        }
        const __half2 zsub = __float2half2_rn(1152.f + zk);      // (c + 1152) - (1152 + zp) = c - zp
#pragma unroll
        for (int c = 0; c < C::KCH; ++c) {
          const uint4 u = *reinterpret_cast<const uint4*>(pg + k_chunk_offset<D * C::ELT>(c, t));
          const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
          if constexpr (C::BF) {
#pragma unroll
            for (int e = 0; e < 4; ++e) w[c * 4 + e] = uw[e];
          } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              uint32_t lo, hi;
              if constexpr (FMT == KVQ_FP8_E4M3) {
                e4m3x4_to_f16x4(uw[e], lo, hi);
              } else {
                const uint32_t x = uw[e] ^ 0x80808080u;          // c + 128 as unsigned bytes
                const uint32_t p0 = __byte_perm(x, 0x64646464u, 0x4140);   // 1024 + byte0|1
                const uint32_t p1 = __byte_perm(x, 0x64646464u, 0x4342);   // 1024 + byte2|3
                __half2 h0 = __hsub2(*reinterpret_cast<const __half2*>(&p0), zsub);
                __half2 h1 = __hsub2(*reinterpret_cast<const __half2*>(&p1), zsub);
                lo = *reinterpret_cast<uint32_t*>(&h0);
                hi = *reinterpret_cast<uint32_t*>(&h1);
              }
              w[c * 8 + 2 * e] = lo;
              w[c * 8 + 2 * e + 1] = hi;
            }
          }
        }
      } else {
#pragma unroll
        for (int i = 0; i < C::KWORDS; ++i) w[i] = 0u;
      }
      const uint32_t col = (j & 1) ? C::COL_AK1 : C::COL_AK0;
#pragma unroll
      for (int c16 = 0; c16 < C::KWORDS / 16; ++c16) {
        uint32_t v16[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) v16[i] = w[c16 * 16 + i];
        tmem_st16(tmem + lane_base + col + 16 * c16, v16);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(akfull + (j & 1));
      mbar_arrive(kempty + s);
      sk_carry = sk;
      valid_carry = mask;
    };

    auto conv_v = [&](int i) {
      const int s = i % C::NST;
      const int tok0 = t0 + 128 * i;
      uint32_t w[64];
      const bool mine = ok && r < D;
#pragma unroll
      for (int p = 0; p < 8; ++p) {
        const int ntok = min(16, max(0, t1 - (tok0 + 16 * p)));
        const bool pv = mine && (valid_cur >> p & 1) && ntok > 0;
        uint32_t pw[8];
        if (pv) {
          const uint8_t* pg = vring + (s * 8 + p) * C::PAGE;
          if constexpr (C::BF) {
            const uint4 u0 = *reinterpret_cast<const uint4*>(pg + r * 16);
            const uint4 u1 = *reinterpret_cast<const uint4*>(pg + D * 16 + r * 16);
            pw[0] = u0.x; pw[1] = u0.y; pw[2] = u0.z; pw[3] = u0.w;
            pw[4] = u1.x; pw[5] = u1.y; pw[6] = u1.z; pw[7] = u1.w;
          } else {
            const uint4 u = *reinterpret_cast<const uint4*>(pg + r * 16);
            const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              if constexpr (FMT == KVQ_FP8_E4M3) {
                e4m3x4_to_f16x4(uw[e], pw[2 * e], pw[2 * e + 1]);
              } else {
                const uint32_t x = uw[e] ^ 0x80808080u;
                const uint32_t p0 = __byte_perm(x, 0x64646464u, 0x4140);
                const uint32_t p1 = __byte_perm(x, 0x64646464u, 0x4342);
                const __half2 k1152 = __float2half2_rn(1152.f);
                __half2 h0 = __hsub2(*reinterpret_cast<const __half2*>(&p0), k1152);
                __half2 h1 = __hsub2(*reinterpret_cast<const __half2*>(&p1), k1152);
                pw[2 * e] = *reinterpret_cast<uint32_t*>(&h0);
                pw[2 * e + 1] = *reinterpret_cast<uint32_t*>(&h1);
              }
            }
          }
          if (ntok < 16) {                                   // tokens past the end -> 0
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const uint32_t keep = (2 * e < ntok ? 0x0000ffffu : 0u) | (2 * e + 1 < ntok ? 0xffff0000u : 0u);
              pw[e] &= keep;
            }
          }
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) pw[e] = 0u;
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) w[p * 8 + e] = pw[e];
      }
#pragma unroll
      for (int c16 = 0; c16 < 4; ++c16) {
        uint32_t v16[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) v16[e] = w[c16 * 16 + e];
        tmem_st16(tmem + lane_base + C::COL_AV + 16 * c16, v16);
      }
      tmem_st_wait();
    };

    auto accum_o = [&](int i) {
      const int s2 = i & 1;
      if (ok) ok = mbar_wait(ofull + s2, (i >> 1) & 1, abort_flag, kWaitLimitCycles);
      tc_fence_after();
      uint32_t oa[16], ob[16];
      if (ok) {
        const uint32_t col = tmem + lane_base + (s2 ? C::COL_O1 : C::COL_O0);
        tmem_ld16(col, oa);
        if constexpr (C::NPR == 32) tmem_ld16(col + 16, ob);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) { oa[e] = 0u; ob[e] = 0u; }
      }
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float v = __uint_as_float(oa[g]) + __uint_as_float(oa[8 + g]);
        if constexpr (C::NPR == 32) v += __uint_as_float(ob[g]);
        o[g] = o[g] * alpha_pend[g] + v * einv_pend;
      }
    };

    conv_k(0);
    for (int i = 0; i < ntiles; ++i) {
      sk_cur = sk_carry;
      valid_cur = valid_carry;
      if (i + 1 < ntiles) conv_k(i + 1);

      // ---- softmax of tile i (thread = token r)
      const int s = i % C::NST;
      if (ok) ok = mbar_wait(vfull + s, (i / C::NST) & 1, abort_flag, kWaitLimitCycles);
      if (ok) ok = mbar_wait(sfull + (i & 1), (i >> 1) & 1, abort_flag, kWaitLimitCycles);
      tc_fence_after();
      uint32_t sw[16];
      if (ok) {
        tmem_ld16(tmem + lane_base + ((i & 1) ? C::COL_S1 : C::COL_S0), sw);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) sw[e] = 0u;
      }
      const int p = r >> 4, t = r & 15;
      const bool valid = ok && (valid_cur >> p & 1) && (t0 + 128 * i + r < t1);
      float sv = 0.f, zv = 0.f;
      if (valid) {
        if constexpr (FMT == KVQ_FP8_E4M3) {
          sv = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(vmeta + (s * 8 + p) * C::METAB)[t]);
        } else if constexpr (FMT == KVQ_INT8_ASYM) {
          const __nv_bfloat16* mm = reinterpret_cast<const __nv_bfloat16*>(vmeta + (s * 8 + p) * C::METAB);
          sv = __bfloat162float(mm[2 * t]);
          zv = __bfloat162float(mm[2 * t + 1]);
        } else {
          sv = 1.f;
        }
      }
      float x[G];
#pragma unroll
      for (int g = 0; g < G; ++g) x[g] = valid ? __uint_as_float(sw[g]) * sk_cur * qs[g] : -INFINITY;
      float* rb = red + (i & 1) * 64;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float tm = warp_max_f32(x[g]);
        if (lane == 0) rb[quarter * 16 + g] = tm;
      }
      {
        const float svm = warp_max_f32(sv);
        if (lane == 0) rb[quarter * 16 + 8] = svm;
      }
      named_bar_sync(1, 128);
      float alpha[G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float tmax = fmaxf(fmaxf(rb[g], rb[16 + g]), fmaxf(rb[32 + g], rb[48 + g]));
        const float mn = fmaxf(m[g], tmax);
        alpha[g] = (mn == -INFINITY) ? 1.f : exp2f(m[g] - mn);
        m[g] = mn;
      }
      const float svmax = fmaxf(fmaxf(rb[8], rb[24]), fmaxf(rb[40], rb[56]));
      int ex = 0;
      if (!C::BF && svmax > 0.f) ex = max(-120, min(120, 14 - ilogbf(svmax)));
      const float escale = __int_as_float((127 + ex) << 23);
      const float einv = __int_as_float((127 - ex) << 23);
      uint8_t* pb = pop + (i & 1) * C::PBYTES;
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float pr = valid ? exp2f(x[g] - m[g]) : 0.f;
        l[g] = l[g] * alpha[g] + pr;
        if constexpr (C::BF) {
          const __nv_bfloat16 hi = __float2bfloat16_rn(pr);
          const float r1 = pr - __bfloat162float(hi);
          const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
          const __nv_bfloat16 lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
          *reinterpret_cast<uint16_t*>(pb + poff[g]) = __bfloat16_as_ushort(hi);
          *reinterpret_cast<uint16_t*>(pb + poff[g] + 1024) = __bfloat16_as_ushort(mid);
          *reinterpret_cast<uint16_t*>(pb + poff[g] + 2048) = __bfloat16_as_ushort(lo);
        } else {
          const float pp = pr * sv * escale;
          const __half hi = __float2half_rn(pp);
          const __half lo = __float2half_rn(pp - __half2float(hi));
          *reinterpret_cast<uint16_t*>(pb + poff[g]) = __half_as_ushort(hi);
          *reinterpret_cast<uint16_t*>(pb + poff[g] + 1024) = __half_as_ushort(lo);
          if constexpr (FMT == KVQ_INT8_ASYM)
            corr[g] = corr[g] * alpha[g] + (__half2float(hi) + __half2float(lo)) * zv * einv;
        }
      }

      // ---- O of the previous tile (its PV is done once ofull flips; AV is free)
      if (i > 0) accum_o(i - 1);
#pragma unroll
      for (int g = 0; g < G; ++g) alpha_pend[g] = alpha[g];
      einv_pend = einv;

      // ---- V of this tile into TMEM, then hand P and V^T to the MMA thread
      conv_v(i);
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(pvready);
      mbar_arrive(vempty + s);
    }
    accum_o(ntiles - 1);

    // ---- chunk partial: (max, sum, unnormalised output) per query head
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float ls = warp_sum(l[g]);
      const float cs = (FMT == KVQ_INT8_ASYM) ? warp_sum(corr[g]) : 0.f;
      if (lane == 0) {
        red2[quarter * 8 + g] = ls;
        red2[32 + quarter * 8 + g] = cs;
      }
    }
    named_bar_sync(1, 128);
    if (ok && !*abort_flag) {
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float L = red2[g] + red2[8 + g] + red2[16 + g] + red2[24 + g];
        const float Cz = red2[32 + g] + red2[40 + g] + red2[48 + g] + red2[56 + g];
        const int64_t row = (int64_t(b) * Hq + h * G + g) * slots + split;
        if (r < D) part_o[row * D + r] = o[g] - Cz;
        if (r == 0) {
          part_ml[row * 2] = m[g];
          part_ml[row * 2 + 1] = L;
        }
      }
      if (r == 0 && split == n_splits - 1) part_cnt[b * Hk + h] = n_splits;
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

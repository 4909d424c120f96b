// attn_fwd_wide.cuh -- the FP8 (e4m3) causal prefill attention forward with
// 256-key KV tiles, Dqk = Dv = 128, for sm_100a.
//
// Method: Zyphra ZYFA, the same steps as attn_fwd.cuh's FP8 path (news pages:
// the-ai.news "Zyphra presenteert ZYFA", section "Drie technieken om de
// bottleneck te omzeilen"; spke.com "Zyphra ZYFA", sections "Lean P" and
// "ブロックごとのスケーリングと丸められた行和"): S = Q K^T in e4m3 with fp32
// accumulation, Lean-P codes with a power-of-two shift per 64-key block, P V
// and the row sum from the rounded codes with block-scaled e4m3 MMAs.
//
// What differs from the 128-key kernel is the tile shape.  An e4m3 MMA of
// M = 128, N = 128, K = 32 with both operands in shared memory runs the
// tensor core well below its rate, one of N = 256 close to it (measured with
// one CTA per SM issuing back to back).  Here S of a tile is one N = 256
// accumulator (256 TMEM columns), so S costs about half the tensor-core time
// per key.  TMEM then holds one S buffer and one P buffer:
//   columns   0-255  S (fp32, 128 rows x 256 keys)
//           256-383  O
//           384-399  row sum l: P V is one N = 144 MMA per 32 keys whose
//                    last 16 columns of B are a shared tile of e4m3 ones,
//                    so columns 384-399 accumulate the row sum of the
//                    rounded, block-scaled P
//           404-411  scale factors of P: keys 0-127 at 404, 128-255 at 408
//                    (row r's E8M0 word in column r / 32 of its own lane)
//           416-447  scale factors of V (E8M0 1.0, wider than N = 144 needs)
//           448-511  P (e4m3 codes, 4 per column): keys 0-127 at 448, 128-255 at 480
// Both softmax warpgroups work on every tile, group x on keys
// 128x .. 128x+127 of it: one thread holds the 128 scores of its row in its
// group's half, read with one TMEM round trip.  A row's tile max is the max of the two
// halves, exchanged once per tile through shared memory under one barrier
// both groups arrive on; both groups then take the same reference-max
// decision, and each codes its half with its own block shifts.
//   warps 0-3   softmax group 0 (keys 0-127 of every tile)
//   warps 4-7   softmax group 1 (keys 128-255 of every tile)
//   warps 8-11  epilogue: O / l -> bf16 -> global, once per unit
//   warp 12     TMA producer: Q tile per unit, K/V ring (32 KB stages)
//   warp 13     S issuer: 4 MMAs of N = 256 per tile
//   warp 14     P V issuer: 8 block-scaled MMAs (K = 32 keys, N = 128 + 16 ones)
//   warp 15     idle (completes the fourth warpgroup for setmaxnreg)
// A unit (batch, query head, 128-row query tile qt) visits KV tiles
// 0 .. qt/2 (integer division); the last one holds the diagonal and, for
// even qt, a second half whose keys all lie after the tile's rows.
#pragma once
#include "attn_fwd.cuh"

namespace zyfa {

struct WideCfg {
  static constexpr int KT = 256;                 // keys per KV tile
  static constexpr int CHUNK = 128 * 128;        // one TMA box: 128 rows x 128 bytes
  static constexpr int QB = CHUNK;               // Q tile: 128 rows x 128 e4m3
  static constexpr int KB = 2 * CHUNK;           // K tile: 256 rows x 128 e4m3
  static constexpr int VB = 2 * CHUNK;           // V tile: 256 rows x 128 e4m3
  static constexpr int STK = 3, STV = 2, QBUF = 2;
  static constexpr int KLEAD = STK - STV + 1;    // K tiles the producer keeps ahead of V
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + QBUF * QB;
  static constexpr int OFF_V = OFF_K + STK * KB;
  static constexpr int OFF_ONES = OFF_V + STV * VB;            // 32 x 128 bytes of e4m3 1.0
  static constexpr int OFF_HAND = OFF_ONES + 4096;             // final reference max per slot x row
  static constexpr int OFF_XCH = OFF_HAND + kHandSlots * 128 * 4;   // half-tile max [2 tiles][2 groups][128]
  static constexpr int OFF_BAR = OFF_XCH + 2 * 2 * 128 * 4;
  // Barriers: QF/QE per Q buffer; OF = O read by the epilogue (per unit);
  // OFIN = last P V of a unit done; SF = S full; SC = S read by both groups;
  // MXA = both groups published their half-tile max; PF = P written by both
  // groups (and O rescaled); PE = P V done (P buffer free, O updated); LF per
  // hand-over slot; KF/KE and VF/VE per ring stage.
  enum { QF0 = 0, QF1, QE0, QE1, OF, OFIN, DRAIN, DRAIN2, SF, SC, MXA, PF, PE, LF0, KF = LF0 + kHandSlots };
  static constexpr int KE = KF + STK, VF = KE + STK, VE = VF + STV;
  static constexpr int NBAR = VE + STV;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;   // + alignment slack
  static constexpr uint32_t TS = 0, TO = 256, TL = 384, TSFB = 416, TSFA = 404, TP = 448;
  static constexpr uint32_t IDESC_QK = idesc_dense(0, 0, 0, 0, 128, 256);
  static_assert(SMEM <= 232448, "shared memory budget");
  // setmaxnreg shares (they add up to the 512 x 128 registers the launch
  // holds): the producer and issuers here hold two ring cursors with their
  // unit iterators, so they get more than in the 128-key kernel, and a
  // softmax thread holds 128 scores plus 32 code words
  static constexpr uint32_t REG_SOFTMAX = 184, REG_EPILOGUE = 80, REG_CONTROL = 64;
  static_assert(128 * (2 * REG_SOFTMAX + REG_EPILOGUE + REG_CONTROL) == kAttnThreads * kLaunchRegs,
                "register split");
};

// EXACTP: the ablation writing P as e4m3(ex2(.)) instead of Lean-P codes.
// VARLEN: packed batch, as in attn_fwd_kernel.
template <bool EXACTP = false, bool VARLEN = false>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_fwd_wide_kernel(const __grid_constant__ AttnArgs a, const __grid_constant__ SeqTable<VARLEN> seqs) {
  const VarlenSeqs* vs = nullptr;
  if constexpr (VARLEN) vs = &seqs;
  using W = WideCfg;
  using TS = TileStream<VARLEN, W::KT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  const uint32_t sb = smem_u32(sm);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  auto bar = [&](int i) -> uint32_t { return sb + W::OFF_BAR + 8u * static_cast<uint32_t>(i); };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sm + W::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + W::OFF_MISC + 4);
  float* hand_m = reinterpret_cast<float*>(sm + W::OFF_HAND);   // [slot][row]
  float* xch_s = reinterpret_cast<float*>(sm + W::OFF_XCH);      // [tile & 1][group][row]

  if (tid == 0) {
    *abort_flag = 0;
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(W::QF0 + i), 1);
      mbar_init(bar(W::QE0 + i), 1);
    }
    mbar_init(bar(W::OF), 128);
    mbar_init(bar(W::OFIN), 1);
    mbar_init(bar(W::DRAIN), 1);
    mbar_init(bar(W::DRAIN2), 1);
    mbar_init(bar(W::SF), 1);
    mbar_init(bar(W::SC), 256);
    mbar_init(bar(W::MXA), 256);
    mbar_init(bar(W::PF), 256);
    mbar_init(bar(W::PE), 1);
    for (int i = 0; i < kHandSlots; ++i) mbar_init(bar(W::LF0 + i), 128);
    for (int i = 0; i < W::STK; ++i) {
      mbar_init(bar(W::KF + i), 1);
      mbar_init(bar(W::KE + i), 1);
    }
    for (int i = 0; i < W::STV; ++i) {
      mbar_init(bar(W::VF + i), 1);
      mbar_init(bar(W::VE + i), 1);
    }
    fence_mbar_init();
  }
  if (warp == 12 && lane == 0) {
    prefetch_tensormap(&a.map_q);
    prefetch_tensormap(&a.map_k);
    prefetch_tensormap(&a.map_v);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_holder), 512);
    tmem_relinquish();
  }
  {
    uint32_t* ones = reinterpret_cast<uint32_t*>(sm + W::OFF_ONES);
    for (int i = tid; i < 1024; i += kAttnThreads) ones[i] = 0x38383838u;   // e4m3 1.0
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_holder;
  const WaitCtl ctl{abort_flag, a.timeout_ns};

  if (warp >= 12) {
   reg_dealloc<W::REG_CONTROL>();
   const bool leader = elect_one();
   const int leader_lane = __ffs(__ballot_sync(0xffffffffu, leader)) - 1;
   auto wait1 = [&](uint32_t br, uint32_t parity) -> bool {
     bool ok = true;
     if (leader) ok = mbar_wait(br, parity, ctl);
     return __shfl_sync(0xffffffffu, ok ? 1 : 0, leader_lane) != 0;
   };
   if (warp == 12) {
    // ------------------------------------------------------------ producer
    // K runs KLEAD tiles ahead of V, in the order the MMAs consume them; a
    // 256-row tile is two 128-row boxes (rows past the tensor read as zero).
    const uint64_t pol_q = l2_policy_evict_first();
    const uint64_t pol_kv = l2_policy_evict_last();
    TS ks, vst;
    ks.init(gridDim.x, blockIdx.x, a, vs);
    vst.init(gridDim.x, blockIdx.x, a, vs);
    bool ok = true;
    int last_q = -1, last_k = -1, last_v = -1;   // last armed unit / tile (abort drain)
    auto load_k = [&](const TS& t) -> bool {
      range_ok(t.b >= 0 && t.b < a.B && t.hq >= 0 && t.hq < a.Hq && t.hkv >= 0 && t.hkv < a.Hkv && t.j >= 0 &&
                   t.j < t.nkv, kChkUnit);
      range_ok(VARLEN ? (t.qt * 128 < t.len && t.r0 >= 0 && t.r0 + t.len <= a.S) : (t.qt * 128 < a.S), kChkRow);
      const int row0 = VARLEN ? t.r0 : 0, tb = VARLEN ? 0 : t.b;
      if (t.j == 0) {
        const uint32_t slot = t.u % W::QBUF, n = t.u / W::QBUF;
        if (n > 0 && !wait1(bar(W::QE0 + slot), (n - 1) & 1)) return false;
        if (leader) {
          mbar_arrive_expect_tx(bar(W::QF0 + slot), W::QB);
          tma_load_4d(sb + W::OFF_Q + slot * W::QB, &a.map_q, bar(W::QF0 + slot), 0, t.hq, row0 + t.qt * 128, tb,
                      pol_q);
        }
        last_q = static_cast<int>(t.u);
      }
      const uint32_t st = t.g % W::STK, n = t.g / W::STK;
      if (n > 0 && !wait1(bar(W::KE + st), (n - 1) & 1)) return false;
      if (leader) {
        mbar_arrive_expect_tx(bar(W::KF + st), W::KB);
#pragma unroll
        for (int h = 0; h < 2; ++h)
          tma_load_4d(sb + W::OFF_K + st * W::KB + h * W::CHUNK, &a.map_k, bar(W::KF + st), 0, t.hkv,
                      row0 + t.j * W::KT + 128 * h, tb, pol_kv);
      }
      last_k = static_cast<int>(t.g);
      __syncwarp();
      return true;
    };
    auto load_v = [&](const TS& t) -> bool {
      const int row0 = VARLEN ? t.r0 : 0, tb = VARLEN ? 0 : t.b;
      const uint32_t st = t.g % W::STV, n = t.g / W::STV;
      if (n > 0 && !wait1(bar(W::VE + st), (n - 1) & 1)) return false;
      if (leader) {
        mbar_arrive_expect_tx(bar(W::VF + st), W::VB);
#pragma unroll
        for (int h = 0; h < 2; ++h)
          tma_load_4d(sb + W::OFF_V + st * W::VB + h * W::CHUNK, &a.map_v, bar(W::VF + st), 0, t.hkv,
                      row0 + t.j * W::KT + 128 * h, tb, pol_kv);
      }
      last_v = static_cast<int>(t.g);
      __syncwarp();
      return true;
    };
    for (int i = 0; i < W::KLEAD && ok && ks.next(); ++i) ok = load_k(ks);
    while (ok && vst.next()) {
      if (ks.next()) ok = load_k(ks);
      if (ok) ok = load_v(vst);
    }
    if (!ok && leader) {
      // let the copies already in flight land before the CTA exits: buffer
      // i's last armed use is the largest index <= last with index % n == i
      auto drain_ring = [&](int last, int n, int bar0) {
        for (int i = 0; i < n && i <= last; ++i) {
          const int x = last - (((last - i) % n) + n) % n;
          drain_wait(bar(bar0 + i), static_cast<uint32_t>(x / n) & 1u, 100000000ull);
        }
      };
      drain_ring(last_q, W::QBUF, W::QF0);
      drain_ring(last_k, W::STK, W::KF);
      drain_ring(last_v, W::STV, W::VF);
    }
    __syncwarp();
   } else if (warp == 13 || warp == 14) {
    // ------------------------------------------------------------ MMA issuers
    // warp 13: S of tile g once its K tile is loaded and both groups have
    // read S of tile g-1 (one S buffer).  warp 14: P V of tile g once both
    // groups have written P (and rescaled O, when the reference moved).
    TS ts;
    ts.init(gridDim.x, blockIdx.x, a, vs);
    bool ok = true;
    const uint64_t dq = smem_desc(sb + W::OFF_Q, 16, 1024, kSw128);
    const uint64_t dk = smem_desc(sb + W::OFF_K, 16, 1024, kSw128);
    auto issue_qk = [&](const TS& t) -> bool {
      const uint32_t slot = t.u % W::QBUF;
      if (t.j == 0 && !wait1(bar(W::QF0 + slot), (t.u / W::QBUF) & 1)) return false;
      const uint32_t st = t.g % W::STK;
      if (!wait1(bar(W::KF + st), (t.g / W::STK) & 1)) return false;
      if (t.g >= 1 && !wait1(bar(W::SC), (t.g - 1) & 1)) return false;
      tc_fence_after();
      if (leader) {
        const uint64_t dqs = dq + ((slot * W::QB) >> 4), dks = dk + ((st * W::KB) >> 4);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_f8_ss(tbase + W::TS, dqs + ((kk * 32) >> 4), dks + ((kk * 32) >> 4), W::IDESC_QK, kk > 0 ? 1u : 0u);
        tc_commit(bar(W::SF));
        tc_commit(bar(W::KE + st));
        if (t.j == t.nkv - 1) tc_commit(bar(W::QE0 + slot));
      }
      __syncwarp();
      return true;
    };
    auto issue_pv = [&](const TS& t) -> bool {
      const uint32_t st = t.g % W::STV;
      const bool first = t.j == 0;
      if (first && t.u > 0 && !wait1(bar(W::OF), (t.u - 1) & 1)) return false;
      if (!wait1(bar(W::VF + st), (t.g / W::STV) & 1)) return false;
      if (!wait1(bar(W::PF), t.g & 1)) return false;   // P stored by both groups, O rescaled
      tc_fence_after();
      if (leader) {
        const uint32_t sfb = tbase + W::TSFB;
        // B of the k-th MMA: V rows 32k .. 32k+31 (MN-major, 128-byte
        // swizzle) as N columns 0-127, and, one leading-byte offset further,
        // the ones tile as columns 128-143
        const uint32_t vst_addr = sb + W::OFF_V + st * W::VB;
#pragma unroll
        for (uint32_t k = 0; k < 8; ++k) {
          const uint32_t k4 = k & 3, sfa = tbase + W::TSFA + 4 * (k >> 2);
          const uint32_t va = vst_addr + k * 4096;
          const uint64_t dvk = smem_desc(va, sb + W::OFF_ONES - va, 1024, kSw128);
          mma_mxf8_ts(tbase + W::TO, tbase + W::TP + 8 * k, dvk, idesc_mxf8(1, 128, 144, k4, k4),
                      sfa | (k4 << 30), sfb | (k4 << 30), (!first || k > 0) ? 1u : 0u);
        }
        tc_commit(bar(W::VE + st));
        tc_commit(bar(W::PE));
        if (t.j == t.nkv - 1) tc_commit(bar(W::OFIN));
      }
      __syncwarp();
      return true;
    };
    if (warp == 13) {
      while (ok && ts.next()) ok = issue_qk(ts);
    } else {
      while (ok && ts.next()) ok = issue_pv(ts);
    }
    if (leader) {
      const uint32_t dr = bar(warp == 13 ? W::DRAIN : W::DRAIN2);
      tc_commit(dr);
      drain_wait(dr, 0, 100000000ull);
    }
    __syncwarp();
   }
  } else if (warp < 8) {
    reg_alloc<W::REG_SOFTMAX>();
    // ------------------------------------------------------------ softmax warpgroups
    // Group x = warp / 4 takes keys 128x .. 128x+127 of every tile; thread t
    // owns row 32 (w % 4) + lane (TMEM lane quarter w % 4).  Per tile: one
    // TMEM read of its half of S (S is free for the next tile once both
    // groups have read it), the two 64-key block maxima, the tile max from
    // both halves, the reference-max decision (the same in both groups), the
    // codes, then, once P V of the previous tile is done, the P store.
    const int grp = warp >> 2;
    const int row = 32 * (warp & 3) + lane;
    const uint32_t lb = tbase + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint32_t tsg = lb + W::TS + 128u * grp;   // this group's half of S
    const uint32_t tpg = lb + W::TP + 32u * grp;    // this group's half of P
    bool ok = true;
    if (grp == 0) {
      for (int c = 0; c < 32; c += 4)   // scale 1.0
        tmem_st4(lb + W::TSFB + c, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu);
      tmem_wait_st();
    }
    TS t;
    t.init(gridDim.x, blockIdx.x, a, vs);
    float A = a.C;
    float m_own = __int_as_float(0xff800000);   // the reference max after the previous tile
    // Two waits per tile are tested early with the non-blocking test_wait and
    // voted on only where the barrier is needed, so the test's latency
    // overlaps other work and a barrier found complete costs no blocking
    // wait: S of the next tile (tested before this tile's P store) and the P
    // buffer (tested before the codes).  A test that finds the phase pending
    // falls back to the bounded wait.  Neither can alias: the phase after the
    // tested one needs work this group has not done yet.
    bool sf_t = false;
    while (ok && t.next()) {
      const uint32_t g = t.g;
      if (t.j == 0) {
        m_own = __int_as_float(0xff800000);
        const bool sok = range_ok(t.b >= 0 && t.b < a.B && t.hq >= 0 && t.hq < a.Hq && t.hkv >= 0 &&
                                  t.hkv < a.Hkv, kChkScale);
        const float qs = (a.q_scale && sok) ? a.q_scale[t.b * a.Hq + t.hq] : 1.0f;
        const float ks = (a.k_scale && sok) ? a.k_scale[t.b * a.Hkv + t.hkv] : 1.0f;
        A = leanp_slope(qs, ks, a.C);
      }
      if (!__all_sync(0xffffffffu, sf_t) && !(ok = warp_wait(bar(W::SF), g & 1, ctl))) break;
      tc_fence_after();
      uint32_t r[128];
      tmem_ld64p(tsg, &r[0]);
      tmem_ld64p(tsg + 64, &r[64]);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(bar(W::SC));
      if (t.j == t.nkv - 1) {
        // key 256 j + 128 grp + c lies after query row 128 qt + row when c > lim
        const int lim = 128 * t.qt + row - W::KT * t.j - 128 * grp;
        if (lim < 127) {
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c > lim) r[c] = 0xff800000u;   // -inf
        }
      }
      const float bmx0 = max64(&r[0]), bmx1 = max64(&r[64]);
      const float hm = fmaxf(bmx0, bmx1);
      // the tile max from both halves (the exchange slot alternates with the
      // tile, and a group reaches tile g+2 only after both arrived for g+1,
      // so a slot is never overwritten before it is read)
      const uint32_t xs = g & 1;
      xch_s[(xs * 2 + grp) * 128 + row] = hm;
      mbar_arrive(bar(W::MXA));
      if (!(ok = warp_wait(bar(W::MXA), g & 1, ctl))) break;
      const float tmax = fmaxf(hm, xch_s[(xs * 2 + (grp ^ 1)) * 128 + row]);
      // reference max after this tile (A carries a factor 8)
      float m, alpha = 1.0f;
      if (t.j == 0) {
        m = tmax;
      } else if (__fmul_rn(tmax - m_own, A) > 8.0f * kRescaleLog2) {
        alpha = ex2_approx(__fmul_rn(__fmul_rn(m_own - tmax, A), 0.125f));
        m = tmax;
      } else {
        m = m_own;
      }
      const bool pe_t = g < 1 || mbar_test_wait(bar(W::PE), (g - 1) & 1);
      // the codes of this group's 128 keys, before waiting for the P buffer
      uint32_t p[32];
      uint32_t sfw = 0;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t* rh = &r[64 * h];
        const int jb = leanp_block_shift(m, h ? bmx1 : bmx0, A);
        if (EXACTP) {
          // p = exp2((s - m) A / 8 + j): one FMA, MUFU ex2, then e4m3
          const float a8 = __fmul_rn(A, 0.125f);
          const float b8 = __fmaf_rn(-m, a8, static_cast<float>(jb));
#pragma unroll
          for (int w = 0; w < 16; ++w) {
            const float e0 = ex2_approx(__fmaf_rn(__uint_as_float(rh[4 * w]), a8, b8));
            const float e1 = ex2_approx(__fmaf_rn(__uint_as_float(rh[4 * w + 1]), a8, b8));
            const float e2 = ex2_approx(__fmaf_rn(__uint_as_float(rh[4 * w + 2]), a8, b8));
            const float e3 = ex2_approx(__fmaf_rn(__uint_as_float(rh[4 * w + 3]), a8, b8));
            p[16 * h + w] = pack_e4m3x2(e0, e1) | (pack_e4m3x2(e2, e3) << 16);
          }
        } else {
          const float Bb = leanp_row_offset(m, A, jb);
          const float a256 = __fmul_rn(A, 0.00390625f), b256 = __fmul_rn(Bb, 0.00390625f);
#pragma unroll
          for (int w = 0; w < 16; ++w) {
            uint32_t w0, w1, w2, w3;
            leanp_code_word2(__uint_as_float(rh[4 * w]), __uint_as_float(rh[4 * w + 1]), a256, b256, w0, w1);
            leanp_code_word2(__uint_as_float(rh[4 * w + 2]), __uint_as_float(rh[4 * w + 3]), a256, b256, w2, w3);
            p[16 * h + w] = pack4_codes(w0, w1, w2, w3);
          }
        }
        // E8M0 scale code 127 - j for both 32-key MX blocks of this 64-key block
        sfw |= static_cast<uint32_t>((127 - jb) * 0x0101) << (16 * h);
      }
      // P V of tile g-1 has read the P buffer and its scale factors, and O holds it
      if (!__all_sync(0xffffffffu, pe_t) && !(ok = warp_wait(bar(W::PE), (g - 1) & 1, ctl))) break;
      tc_fence_after();
      if (__any_sync(0xffffffffu, alpha != 1.0f)) {
        // the reference moved: O and l still hold tiles 0 .. g-1 against the
        // old one; each group rescales its 64 columns of O, group 0 also l
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          uint32_t o[32];
          tmem_ld32p(lb + W::TO + 64 * grp + 32 * q, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32p(lb + W::TO + 64 * grp + 32 * q, o);
        }
        if (grp == 0) {
          const uint32_t lv = tmem_ld1(lb + W::TL);
          tmem_wait_ld();
          tmem_st1(lb + W::TL, __float_as_uint(__uint_as_float(lv) * alpha));
        }
      }
      sf_t = mbar_test_wait(bar(W::SF), (g + 1) & 1);
      tmem_st16p(tpg, &p[0]);
      tmem_st16p(tpg + 16, &p[16]);
      // the row's E8M0 word of this half: column (row / 32) of its own lane
      tmem_st1(lb + W::TSFA + 4 * grp + (warp & 3), sfw);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(W::PF));
      m_own = m;
      if (t.j == t.nkv - 1 && grp == 0) {
        // the unit's final reference max, for the epilogue's log-sum-exp
        const uint32_t hs = t.u % kHandSlots;
        hand_m[hs * 128 + row] = m;
        mbar_arrive(bar(W::LF0 + hs));
      }
    }
  } else {
    reg_dealloc<W::REG_EPILOGUE>();
    // ------------------------------------------------------------ epilogue warpgroup
    const int row = 32 * (warp & 3) + lane;
    const uint32_t lb = tbase + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    typename std::conditional<VARLEN, VarlenIter, UnitIter>::type units;
    if constexpr (VARLEN) units.init(gridDim.x, blockIdx.x, vs, a.Hq, a.Hkv);
    else units.init(gridDim.x, blockIdx.x, a.Tq, a.Hq, a.Hkv, a.B, a.group_slots);
    uint32_t u_it = 0;
    int b, hkv, hq, qt;
    int r0 = 0, len = 0;
    bool ok = true;
    while (ok && (VARLEN ? units.next(b, hkv, hq, qt, r0, len) : units.next(b, hkv, hq, qt))) {
      if (!(ok = warp_wait(bar(W::OFIN), u_it & 1, ctl))) break;
      const uint32_t hs = u_it % kHandSlots;
      if (!(ok = warp_wait(bar(W::LF0 + hs), (u_it / kHandSlots) & 1, ctl))) break;
      tc_fence_after();
      const float m_last = hand_m[hs * 128 + row];
      const int grow = qt * 128 + row;
      const bool sok = range_ok(b >= 0 && b < a.B && hq >= 0 && hq < a.Hq && hkv >= 0 && hkv < a.Hkv, kChkScale);
      const float vsc = (a.v_scale && sok) ? a.v_scale[b * a.Hkv + hkv] : 1.0f;
      const float lv = __uint_as_float(tmem_ld1(lb + W::TL));
      tmem_wait_ld();
      const float inv = vsc / lv;
      float lse_log2 = 0.0f;
      if (a.lse) {   // weights are 2^((s - m) A / 8) against the final reference m
        const float qs = (a.q_scale && sok) ? a.q_scale[b * a.Hq + hq] : 1.0f;
        const float ks = (a.k_scale && sok) ? a.k_scale[b * a.Hkv + hkv] : 1.0f;
        const float A8 = __fmul_rn(leanp_slope(qs, ks, a.C), 0.125f);
        lse_log2 = __fmaf_rn(m_last, A8, log2f(lv));
      }
      const bool wok = range_ok(grow >= (VARLEN ? len : a.S) ||
                                    (hq >= 0 && hq < a.Hq &&
                                     (VARLEN ? (r0 >= 0 && r0 + grow < a.S) : (b >= 0 && b < a.B))),
                                kChkStore);
      __nv_bfloat16* orow;
      if constexpr (VARLEN) {
        if (a.lse && grow < len && wok)
          a.lse[static_cast<size_t>(hq) * a.S + r0 + grow] = lse_log2 * 0.69314718055994530942f;
        orow = a.o + ((static_cast<size_t>(r0) + grow) * a.Hq + hq) * 128;
      } else {
        if (a.lse && grow < a.S && wok)
          a.lse[(static_cast<size_t>(b) * a.Hq + hq) * a.S + grow] = lse_log2 * 0.69314718055994530942f;
        orow = a.o + ((static_cast<size_t>(b) * a.S + grow) * a.Hq + hq) * 128;
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t o[32];
        tmem_ld32p(lb + W::TO + 32 * q, o);
        tmem_wait_ld();
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          w[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
        if (grow < (VARLEN ? len : a.S) && wok) {
          uint4* dst = reinterpret_cast<uint4*>(orow + 32 * q);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
        }
      }
      tc_fence_before();
      mbar_arrive(bar(W::OF));
      ++u_it;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tbase, 512);
}

}  // namespace zyfa

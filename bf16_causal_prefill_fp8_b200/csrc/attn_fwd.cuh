// attn_fwd.cuh -- causal prefill attention forward, O = softmax(Q K^T * scale
// + causal mask) V, for sm_100a: persistent causal-aware scheduler, TMA-staged
// K/V ring, tcgen05 MMAs into tensor memory, a warp-specialised softmax.
//
// Method: Zyphra ZYFA (news pages: the-ai.news "Zyphra presenteert ZYFA",
// sections "Waarom presteert FP8 minder goed op de MI355X?" and "Drie
// technieken om de bottleneck te omzeilen"; spke.com "Zyphra ZYFA", sections
// "Lean P", "2ウェーブのピンポンスケジュール", "ブロックごとのスケーリングと丸
// められた行和"; kongchang.com "Zyphra ZYFA", FlashAttention tiling with an
// online softmax).  FP8 path: Q K^T in e4m3, P written Lean-P style as e4m3
// codes with a power-of-two scale per 64-key block, P V and the row sum taken
// with block-scaled e4m3 MMAs that remove the scale.  BF16 path: the same
// pipeline with exact exp2 probabilities rounded to bf16.
//
// CTA = 192 threads, one per SM (persistent grid):
//   warps 0-3  softmax warpgroup: thread t owns query row t of the tile and
//              TMEM lane t; online max, P, O rescale, epilogue
//   warp 4     TMA producer (one thread): Q tile once per unit, K/V ring
//   warp 5     MMA issuer (one thread): S = Q K^T, O += P V (+ row sum)
// Work unit = (batch, query head, 128-row query tile); KV tiles 0..qt only
// (fully masked tiles are never issued), ascending, so results are
// deterministic.  The MMA for S of tile j+1 overlaps the softmax of tile j
// (two S buffers in TMEM); the P V MMA of tile j overlaps the softmax of
// tile j+1.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "leanp.cuh"
#include "ptx.cuh"

namespace zyfa {

struct AttnArgs {
  CUtensorMap map_q;       // 128-byte column chunk boxes of Q (128 rows), 128-byte swizzle
  CUtensorMap map_q_tail;  // FP8 with Dqk 192: the 64-byte tail box, 64-byte swizzle
  CUtensorMap map_k;
  CUtensorMap map_k_tail;
  CUtensorMap map_v;
  __nv_bfloat16* o;
  const float* q_scale;    // [B*Hq] or null (1.0); FP8 only
  const float* k_scale;    // [B*Hkv] or null
  const float* v_scale;    // [B*Hkv] or null
  int B, Hq, Hkv, S;
  int Tq;                  // query tiles per head, ceil(S / 128)
  int group_slots;         // (batch, kv head) slots per scheduling group
  float C;                 // FP8: 8 log2(e)/sqrt(Dqk); BF16: log2(e)/sqrt(Dqk)
  unsigned long long timeout_ns;
};

template <bool FP8, int DQK>
struct AttnCfg {
  static constexpr int EL = FP8 ? 1 : 2;            // bytes per input element
  static constexpr int ROWB = DQK * EL;              // bytes per Q/K row
  static constexpr int NCH = ROWB / 128;             // 128-byte swizzled column chunks
  static constexpr bool TAIL = (ROWB % 128) != 0;    // FP8 Dqk 192: one 64-byte chunk more
  static constexpr int CHUNK = 128 * 128;            // bytes of one 128-row, 128-byte chunk
  static constexpr int QB = 128 * ROWB;
  static constexpr int KB = 128 * ROWB;
  static constexpr int VB = 128 * 128 * EL;          // Dv = 128
  static constexpr int ST = FP8 ? 4 : 2;             // K/V ring stages
  static constexpr int NK_QK = ROWB / 32;            // QK MMA K-steps of 32 bytes
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + QB;
  static constexpr int OFF_V = OFF_K + ST * KB;
  static constexpr int OFF_ONES = OFF_V + ST * VB;   // FP8: 16 x 128 bytes of e4m3 1.0
  static constexpr int OFF_SFX = OFF_ONES + (FP8 ? 2048 : 0);
  static constexpr int OFF_BAR = OFF_SFX + 2 * 128 * 4;
  enum { QF = 0, QE, OD, OF, DRAIN, SF0, SF1, SC0, SC1, PF0, PF1, SX0, SX1, KF, };
  static constexpr int KE = KF + ST, VF = KF + 2 * ST, VE = KF + 3 * ST;
  static constexpr int NBAR = KF + 4 * ST;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;  // + alignment slack
  // tensor-memory columns (512 allocated)
  static constexpr uint32_t TS0 = 0, TS1 = 128, TO = 256;
  static constexpr uint32_t TL = 384, TSFB = 400, TSFA0 = 404, TSFA1 = 408;
  static constexpr uint32_t TP0 = FP8 ? 448 : 384, TP1 = FP8 ? 480 : 448;
  static constexpr uint32_t IDESC_QK = idesc_dense(FP8 ? 0 : 1, FP8 ? 0 : 1, 0, 0, 128, 128);
  static constexpr uint32_t IDESC_PV_BF16 = idesc_dense(1, 1, 0, 1, 128, 128);
  static_assert(SMEM <= 232448, "shared memory budget");
};

// Static causal-aware schedule.  Units are grouped by (batch, kv head) slots so
// that one group's K/V stays resident in L2; inside a group the heaviest query
// tiles (most KV tiles) come first, and consecutive units share a kv head.
// Units are dealt round-robin to the persistent CTAs, reversing direction on
// every round so per-CTA work evens out.
struct UnitIter {
  int G, c, Tq, gq, Hkv, slots, Gk, ngroups;
  int g, k, slots_g, U_g;
  __device__ void init(int grid, int cta, int Tq_, int Hq, int Hkv_, int B, int Gk_) {
    G = grid; c = cta; Tq = Tq_; Hkv = Hkv_; gq = Hq / Hkv_;
    slots = B * Hkv_; Gk = Gk_; ngroups = (slots + Gk - 1) / Gk;
    g = 0; k = 0;
    slots_g = min(Gk, slots); U_g = slots_g * gq * Tq;
  }
  __device__ bool next(int& b, int& hkv, int& hq, int& qt) {
    while (g < ngroups) {
      if (k * G >= U_g) {
        ++g; k = 0;
        if (g < ngroups) { slots_g = min(Gk, slots - g * Gk); U_g = slots_g * gq * Tq; }
        continue;
      }
      const int p = k * G + ((k & 1) ? (G - 1 - c) : c);
      ++k;
      if (p >= U_g) continue;
      const int per = slots_g * gq;
      const int r = p / per, rem = p - r * per;
      qt = Tq - 1 - r;
      const int slot = g * Gk + rem / gq;
      b = slot / Hkv;
      hkv = slot - b * Hkv;
      hq = hkv * gq + (rem - (rem / gq) * gq);
      return true;
    }
    return false;
  }
};

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Two fp32 values -> bf16x2 (round to nearest even), first value in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}

__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, const WaitCtl& ctl) {
  const bool ok = mbar_wait(bar, parity, ctl);
  return __all_sync(0xffffffffu, ok);
}

// Wait ignoring the abort flag, for draining in-flight work before exit.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > limit_ns) {
      atomicExch(&g_device_status, kDevWaitTimeout);
      return;
    }
  }
}

// Max of 64 consecutive fp32 values (held as bits) with 8 independent chains.
__device__ __forceinline__ float max64(const uint32_t* s) {
  float a[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) a[i] = __uint_as_float(s[i]);
#pragma unroll
  for (int c = 8; c < 64; c += 8)
#pragma unroll
    for (int i = 0; i < 8; ++i) a[i] = fmaxf(a[i], __uint_as_float(s[c + i]));
  return fmaxf(fmaxf(fmaxf(a[0], a[1]), fmaxf(a[2], a[3])), fmaxf(fmaxf(a[4], a[5]), fmaxf(a[6], a[7])));
}

template <bool FP8, int DQK>
__global__ void __launch_bounds__(192, 1) attn_fwd_kernel(const __grid_constant__ AttnArgs a) {
  using Cf = AttnCfg<FP8, DQK>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  const uint32_t sb = smem_u32(sm);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  auto bar = [&](int i) -> uint32_t { return sb + Cf::OFF_BAR + 8u * static_cast<uint32_t>(i); };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sm + Cf::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + Cf::OFF_MISC + 4);
  uint32_t* sfx = reinterpret_cast<uint32_t*>(sm + Cf::OFF_SFX);

  if (tid == 0) {
    *abort_flag = 0;
    mbar_init(bar(Cf::QF), 1);
    mbar_init(bar(Cf::QE), 1);
    mbar_init(bar(Cf::OD), 1);
    mbar_init(bar(Cf::OF), 128);
    mbar_init(bar(Cf::DRAIN), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(Cf::SF0 + i), 1);
      mbar_init(bar(Cf::SC0 + i), 128);
      mbar_init(bar(Cf::PF0 + i), 128);
      mbar_init(bar(Cf::SX0 + i), 128);
    }
    for (int i = 0; i < Cf::ST; ++i) {
      mbar_init(bar(Cf::KF + i), 1);
      mbar_init(bar(Cf::KE + i), 1);
      mbar_init(bar(Cf::VF + i), 1);
      mbar_init(bar(Cf::VE + i), 1);
    }
    fence_mbar_init();
  }
  if (warp == 4 && lane == 0) {
    prefetch_tensormap(&a.map_q);
    prefetch_tensormap(&a.map_k);
    prefetch_tensormap(&a.map_v);
    if (Cf::TAIL) { prefetch_tensormap(&a.map_q_tail); prefetch_tensormap(&a.map_k_tail); }
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_holder), 512);
    tmem_relinquish();
  }
  if (FP8) {
    uint32_t* ones = reinterpret_cast<uint32_t*>(sm + Cf::OFF_ONES);
    for (int i = tid; i < 512; i += 192) ones[i] = 0x38383838u;   // e4m3 1.0
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_holder;
  const WaitCtl ctl{abort_flag, a.timeout_ns};
  UnitIter units;
  units.init(gridDim.x, blockIdx.x, a.Tq, a.Hq, a.Hkv, a.B, a.group_slots);
  const int gq = a.Hq / a.Hkv;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol_q = l2_policy_evict_first();
      const uint64_t pol_kv = l2_policy_evict_last();
      uint32_t kv_it = 0, u_it = 0;
      int b, hkv, hq, qt;
      bool ok = true;
      auto load_qk = [&](uint32_t dst, const CUtensorMap* m, const CUtensorMap* mt, uint32_t br,
                         int h, int row, int bb, uint64_t pol) {
#pragma unroll
        for (int c = 0; c < Cf::NCH; ++c)
          tma_load_4d(dst + c * Cf::CHUNK, m, br, c * (128 / Cf::EL), h, row, bb, pol);
        if (Cf::TAIL) tma_load_4d(dst + Cf::NCH * Cf::CHUNK, mt, br, 128, h, row, bb, pol);
      };
      while (ok && units.next(b, hkv, hq, qt)) {
        if (u_it > 0 && !(ok = mbar_wait(bar(Cf::QE), (u_it - 1) & 1, ctl))) break;
        mbar_arrive_expect_tx(bar(Cf::QF), Cf::QB);
        load_qk(sb + Cf::OFF_Q, &a.map_q, &a.map_q_tail, bar(Cf::QF), hq, qt * 128, b, pol_q);
        for (int j = 0; j <= qt; ++j, ++kv_it) {
          const uint32_t st = kv_it % Cf::ST, n = kv_it / Cf::ST;
          if (n > 0 && !(ok = mbar_wait(bar(Cf::KE + st), (n - 1) & 1, ctl))) break;
          mbar_arrive_expect_tx(bar(Cf::KF + st), Cf::KB);
          load_qk(sb + Cf::OFF_K + st * Cf::KB, &a.map_k, &a.map_k_tail, bar(Cf::KF + st), hkv,
                  j * 128, b, pol_kv);
          if (n > 0 && !(ok = mbar_wait(bar(Cf::VE + st), (n - 1) & 1, ctl))) break;
          mbar_arrive_expect_tx(bar(Cf::VF + st), Cf::VB);
#pragma unroll
          for (int c = 0; c < Cf::VB / Cf::CHUNK; ++c)
            tma_load_4d(sb + Cf::OFF_V + st * Cf::VB + c * Cf::CHUNK, &a.map_v, bar(Cf::VF + st),
                        c * (128 / Cf::EL), hkv, j * 128, b, pol_kv);
        }
        ++u_it;
      }
      if (!ok) {
        // let copies already in flight land before the CTA exits
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 200000ull) __nanosleep(1000);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t qk_it = 0, u_it = 0;
      int b, hkv, hq, qt;
      bool ok = true;
      auto issue_pv = [&](uint32_t kvi, bool first) -> bool {
        const uint32_t st = kvi % Cf::ST, buf = kvi & 1;
        if (!mbar_wait(bar(Cf::PF0 + buf), (kvi >> 1) & 1, ctl)) return false;
        if (!mbar_wait(bar(Cf::VF + st), (kvi / Cf::ST) & 1, ctl)) return false;
        if (first && u_it > 0 && !mbar_wait(bar(Cf::OF), (u_it - 1) & 1, ctl)) return false;
        tc_fence_after();
        const uint32_t vbase = sb + Cf::OFF_V + st * Cf::VB;
        const uint32_t tp = tbase + (buf ? Cf::TP1 : Cf::TP0);
        if (FP8) {
          const uint32_t sfa = tbase + (buf ? Cf::TSFA1 : Cf::TSFA0);
          const uint32_t sfb = tbase + Cf::TSFB;
#pragma unroll
          for (uint32_t ks = 0; ks < 4; ++ks) {
            const uint64_t bd = smem_desc(vbase + ks * 4096, 16384, 1024, kSw128);
            mma_mxf8_ts(tbase + Cf::TO, tp + 8 * ks, bd, idesc_mxf8(1, 128, 128, ks, ks),
                        sfa | (ks << 30), sfb | (ks << 30), (!first || ks > 0) ? 1u : 0u);
          }
#pragma unroll
          for (uint32_t ks = 0; ks < 4; ++ks) {
            const uint64_t bd = smem_desc(sb + Cf::OFF_ONES + ks * 32, 16, 1024, kSw128);
            mma_mxf8_ts(tbase + Cf::TL, tp + 8 * ks, bd, idesc_mxf8(0, 128, 16, ks, ks),
                        sfa | (ks << 30), sfb | (ks << 30), (!first || ks > 0) ? 1u : 0u);
          }
        } else {
#pragma unroll
          for (uint32_t ks = 0; ks < 8; ++ks) {
            const uint64_t bd = smem_desc(vbase + ks * 2048, 16384, 1024, kSw128);
            mma_f16_ts(tbase + Cf::TO, tp + 8 * ks, bd, Cf::IDESC_PV_BF16,
                       (!first || ks > 0) ? 1u : 0u);
          }
        }
        tc_commit(bar(Cf::OD));
        tc_commit(bar(Cf::VE + st));
        return true;
      };
      while (ok && units.next(b, hkv, hq, qt)) {
        const int nkv = qt + 1;
        if (!(ok = mbar_wait(bar(Cf::QF), u_it & 1, ctl))) break;
        for (int j = 0; j < nkv && ok; ++j) {
          const uint32_t kvi = qk_it + j, st = kvi % Cf::ST, buf = kvi & 1;
          if (!(ok = mbar_wait(bar(Cf::KF + st), (kvi / Cf::ST) & 1, ctl))) break;
          if (kvi >= 2 && !(ok = mbar_wait(bar(Cf::SC0 + buf), ((kvi >> 1) - 1) & 1, ctl))) break;
          tc_fence_after();
          const uint32_t kbase = sb + Cf::OFF_K + st * Cf::KB;
          const uint32_t ts = tbase + (buf ? Cf::TS1 : Cf::TS0);
#pragma unroll
          for (int kk = 0; kk < Cf::NK_QK; ++kk) {
            uint32_t off, sbo, swz;
            if (kk < Cf::NCH * 4) { off = (kk >> 2) * Cf::CHUNK + (kk & 3) * 32; sbo = 1024; swz = kSw128; }
            else { off = Cf::NCH * Cf::CHUNK + (kk - Cf::NCH * 4) * 32; sbo = 512; swz = kSw64; }
            const uint64_t ad = smem_desc(sb + Cf::OFF_Q + off, 16, sbo, swz);
            const uint64_t bd = smem_desc(kbase + off, 16, sbo, swz);
            if (FP8) mma_f8_ss(ts, ad, bd, Cf::IDESC_QK, kk > 0 ? 1u : 0u);
            else mma_f16_ss(ts, ad, bd, Cf::IDESC_QK, kk > 0 ? 1u : 0u);
          }
          tc_commit(bar(Cf::SF0 + buf));
          tc_commit(bar(Cf::KE + st));
          if (j == nkv - 1) tc_commit(bar(Cf::QE));
          if (j >= 1) ok = issue_pv(kvi - 1, j == 1);
        }
        if (ok) ok = issue_pv(qk_it + nkv - 1, nkv == 1);
        qk_it += nkv;
        ++u_it;
      }
      // all MMAs issued by this thread must finish before TMEM is released
      tc_commit(bar(Cf::DRAIN));
      drain_wait(bar(Cf::DRAIN), 0, 100000000ull);
    }
  } else {
    // ------------------------------------------------------------ softmax warpgroup
    const int row = tid;   // query row inside the tile == TMEM lane
    const uint32_t lb = tbase + (static_cast<uint32_t>(warp * 32) << 16);
    uint32_t kv_it = 0, u_it = 0;
    int b, hkv, hq, qt;
    bool ok = true;
    if (FP8) {
      tmem_st4(lb + Cf::TSFB, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu);  // scale 1.0
      tmem_wait_st();
    }
    while (ok && units.next(b, hkv, hq, qt)) {
      const int nkv = qt + 1;
      float A = a.C, vsc = 1.0f;
      if (FP8) {
        const float qs = a.q_scale ? a.q_scale[b * a.Hq + hq] : 1.0f;
        const float ks = a.k_scale ? a.k_scale[b * a.Hkv + hkv] : 1.0f;
        vsc = a.v_scale ? a.v_scale[b * a.Hkv + hkv] : 1.0f;
        A = leanp_slope(qs, ks, a.C);
      }
      float m = __int_as_float(0xff800000);
      float l = 0.0f;
      for (int j = 0; j < nkv; ++j, ++kv_it) {
        const uint32_t buf = kv_it & 1;
        if (!(ok = warp_wait(bar(Cf::SF0 + buf), (kv_it >> 1) & 1, ctl))) break;
        tc_fence_after();
        uint32_t r[128];
        {
          const uint32_t ts = lb + (buf ? Cf::TS1 : Cf::TS0);
          tmem_ld32p(ts, &r[0]);
          tmem_ld32p(ts + 32, &r[32]);
          tmem_ld32p(ts + 64, &r[64]);
          tmem_ld32p(ts + 96, &r[96]);
          tmem_wait_ld();
        }
        tc_fence_before();
        mbar_arrive(bar(Cf::SC0 + buf));
        if (j == qt) {
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c > row) r[c] = 0xff800000u;   // -inf: key after the query row
        }
        const float bm0 = max64(r), bm1 = max64(r + 64);
        const float m_new = fmaxf(m, fmaxf(bm0, bm1));
        uint32_t p[32];
        float tile_sum = 0.0f;
        uint32_t sf0 = 0, sf1 = 0, sf2 = 0, sf3 = 0;
        if (FP8) {
          const int j0 = leanp_block_shift(m_new, bm0, A);
          const int j1 = leanp_block_shift(m_new, bm1, A);
          const float B0 = leanp_row_offset(m_new, A, j0);
          const float B1 = leanp_row_offset(m_new, A, j1);
#pragma unroll
          for (int w = 0; w < 32; ++w) {
            const float Bw = w < 16 ? B0 : B1;
            p[w] = pack4_low_bytes(leanp_code_word(__uint_as_float(r[4 * w]), A, Bw),
                                   leanp_code_word(__uint_as_float(r[4 * w + 1]), A, Bw),
                                   leanp_code_word(__uint_as_float(r[4 * w + 2]), A, Bw),
                                   leanp_code_word(__uint_as_float(r[4 * w + 3]), A, Bw));
          }
          // E8M0 scale codes 127 - j: bytes 0,1 cover keys 0-63, bytes 2,3 keys 64-127
          const uint32_t e0 = static_cast<uint32_t>(127 - j0), e1 = static_cast<uint32_t>(127 - j1);
          sfx[buf * 128 + row] = e0 * 0x0101u | (e1 * 0x0101u) << 16;
          mbar_arrive(bar(Cf::SX0 + buf));
          if (!(ok = warp_wait(bar(Cf::SX0 + buf), (kv_it >> 1) & 1, ctl))) break;
          // scale-factor layout for M = 128: column c, lane 32w+i holds row 32c+i (all w)
          sf0 = sfx[buf * 128 + lane];
          sf1 = sfx[buf * 128 + 32 + lane];
          sf2 = sfx[buf * 128 + 64 + lane];
          sf3 = sfx[buf * 128 + 96 + lane];
        } else {
          const float mc = m_new * A;
          float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
          uint32_t pb[64];
#pragma unroll
          for (int w = 0; w < 64; ++w) {
            const float p0 = ex2_approx(__fmaf_rn(__uint_as_float(r[2 * w]), A, -mc));
            const float p1 = ex2_approx(__fmaf_rn(__uint_as_float(r[2 * w + 1]), A, -mc));
            acc[w & 3] += p0 + p1;
            pb[w] = pack_bf16x2(p0, p1);
          }
          tile_sum = (acc[0] + acc[1]) + (acc[2] + acc[3]);
          const uint32_t tp = lb + (buf ? Cf::TP1 : Cf::TP0);
          tmem_st32p(tp, &pb[0]);
          tmem_st32p(tp + 32, &pb[32]);
        }
        // online-softmax correction of O (and l) when the running max grew
        if (j > 0) {
          const bool need = m_new > m;
          const float alpha = need ? ex2_approx(__fmul_rn(__fmul_rn(m - m_new, A), FP8 ? 0.125f : 1.0f)) : 1.0f;
          if (!FP8) l *= alpha;
          if (__any_sync(0xffffffffu, need)) {
            if (!(ok = warp_wait(bar(Cf::OD), (kv_it - 1) & 1, ctl))) break;
            tc_fence_after();
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint32_t o[32];
              tmem_ld32p(lb + Cf::TO + 32 * q, o);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
              tmem_st32p(lb + Cf::TO + 32 * q, o);
            }
            if (FP8) {
              const uint32_t lv = tmem_ld1(lb + Cf::TL);
              tmem_wait_ld();
              tmem_st1(lb + Cf::TL, __float_as_uint(__uint_as_float(lv) * alpha));
            }
          }
        }
        if (!FP8) l += tile_sum;
        m = m_new;
        if (FP8) {
          const uint32_t tp = lb + (buf ? Cf::TP1 : Cf::TP0);
          tmem_st32p(tp, p);
          tmem_st4(lb + (buf ? Cf::TSFA1 : Cf::TSFA0), sf0, sf1, sf2, sf3);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(Cf::PF0 + buf));
      }
      if (!ok) break;
      // ---- epilogue: O / l (* v_scale) -> bf16, rows past S are not written
      if (!(ok = warp_wait(bar(Cf::OD), (kv_it - 1) & 1, ctl))) break;
      tc_fence_after();
      float inv;
      if (FP8) {
        const float lv = __uint_as_float(tmem_ld1(lb + Cf::TL));
        tmem_wait_ld();
        inv = vsc / lv;
      } else {
        inv = 1.0f / l;
      }
      const int grow = qt * 128 + row;
      __nv_bfloat16* orow = a.o + ((static_cast<size_t>(b) * a.S + grow) * a.Hq + hq) * 128;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t o[32];
        tmem_ld32p(lb + Cf::TO + 32 * q, o);
        tmem_wait_ld();
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          w[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
        if (grow < a.S) {
          uint4* dst = reinterpret_cast<uint4*>(orow + 32 * q);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
        }
      }
      tc_fence_before();
      mbar_arrive(bar(Cf::OF));
      ++u_it;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tbase, 512);
  (void)gq;
}

}  // namespace zyfa

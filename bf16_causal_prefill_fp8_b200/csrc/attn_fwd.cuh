// attn_fwd.cuh -- causal prefill attention forward, O = softmax(Q K^T * scale
// + causal mask) V, for sm_100a: persistent causal-aware scheduler, TMA-staged
// K/V ring, tcgen05 MMAs into tensor memory, warp-specialised softmax.
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
// The pages overlap matrix and vector work by instruction order (two waves
// per SIMD, ping-pong).  Blackwell tracks MMA completion in hardware, so the
// overlap here is warp specialisation with mbarrier hand-offs.  CTA = 512
// threads (four warpgroups), one per SM (persistent grid); setmaxnreg moves
// registers to the softmax warpgroups, which hold a whole 128-key row of S:
//   warps 0-7   softmax, two warpgroups taking alternate KV tiles
//               (ping-pong): warp w owns rows 32(w%4) .. 32(w%4)+31 of the
//               tile (TMEM lane quarter w%4), all 128 keys.  Per tile: one
//               TMEM read of S (the S buffer is released at once), reference
//               max (handed from group to group), P (Lean-P codes or bf16),
//               and, when the reference max moved, the O rescale of its rows
//   warps 8-11  epilogue: O / l -> bf16 -> global, once per unit
//   warp 12     TMA producer (one elected thread): Q tile per unit, K/V ring
//   warp 13     S issuer (one elected thread): S = Q K^T
//   warp 14     P V issuer (one elected thread): O += P V (+ the FP8 row sum)
//   warp 15     idle (completes the fourth warpgroup for setmaxnreg)
// The two MMA streams are issued by different warps so that S of a later
// tile never queues behind P V of an earlier one (each warp commits only its
// own MMAs; the hand-offs between them go through the barriers).
// Work unit = (batch, query head, 128-row query tile); KV tiles 0..qt only
// (fully masked tiles are never issued), ascending, so results are
// deterministic.  FP8 and BF16 with Dqk 192: S has two TMEM buffers, and the
// MMA of S for tile j+2 runs as soon as the softmax has read S of tile j.
// BF16 with Dqk 128: Q sits in TMEM (copied from shared memory once per unit
// with tcgen05.cp) and S is a TS MMA, A from TMEM and only K from shared
// memory; with both operands in shared memory the N = 128 MMA is bound by
// shared-memory bandwidth.  Q takes the second S buffer's columns, so S of
// tile j+1 runs as soon as the softmax has read S of tile j.  P V of tile j
// runs while the softmax works on tile j+1.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>
#include <type_traits>

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
  float* lse;              // [B, Hq, S] natural-log sum of exp(scaled scores) per row, or null
  const float* q_scale;    // [B*Hq] or null (1.0); FP8 only
  const float* k_scale;    // [B*Hkv] or null
  const float* v_scale;    // [B*Hkv] or null
  int B, Hq, Hkv, S;
  int Tq;                  // query tiles per head, ceil(S / 128)
  int group_slots;         // (batch, kv head) slots per scheduling group
  float C;                 // FP8: 8 log2(e)/sqrt(Dqk); BF16: log2(e)/sqrt(Dqk)
  unsigned long long timeout_ns;
};

constexpr int kAttnThreads = 512;
// Register split (setmaxnreg; the launch holds 512 x 128 = 65536 registers,
// the whole register file, and the four shares below add up to it; zyfa.cu
// checks the compiled count before the first launch, since a raise that asks
// for more than the launch holds would wait forever): softmax warpgroups
// hold a 128-key row of S plus its codes, the epilogue warpgroup one
// 32-column slice of O, the producer / issuer warpgroup only loop state.
constexpr uint32_t kRegSoftmax = 192, kRegEpilogue = 80, kRegControl = 48;
constexpr int kLaunchRegs = 128;
static_assert(128 * (2 * kRegSoftmax + kRegEpilogue + kRegControl) == kAttnThreads * kLaunchRegs,
              "register split");
// Deferred reference max (both paths): the max that the probabilities are
// taken against moves only when a tile's max exceeds it by more than this
// many binades (FlashAttention-4's lazy rescale, with a far larger bound).
// O and the row sum always share the reference, so the softmax is unchanged,
// and the O rescale, which makes P V of a tile wait for P V of the previous
// one, becomes rare.  The bound is set by number range, not precision: FP8
// renormalises every 64-key block to its own max with the shift j (its top
// code stays in (112, 120]), so a block above the reference only takes j down
// to 8 - kRescaleLog2 and an E8M0 scale 2^(kRescaleLog2 - 8) > 1; BF16 P
// values reach 2^kRescaleLog2, inside bf16's range.  Weights <= 2^64 keep O
// (at most 2^64 * 448 * 2^17 for S <= 2^17) and the row sum far inside fp32.
constexpr float kRescaleLog2 = 64.0f;
static_assert(kRescaleLog2 <= 100.0f, "E8M0 scale range and fp32 accumulator headroom");
// Unit hand-overs from the softmax warpgroups to the epilogue (the final
// reference max, and for BF16 each group's partial row sum) go through a ring
// of this many slots, each with its own barrier.  A group can get ahead of
// the epilogue by at most P-buffer count + 2 units (its P buffer waits tie it
// to P V, and P V of the next unit waits for the epilogue), so 8 > 3 + 2.
constexpr int kHandSlots = 8;

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
  // ring stages: FP8 4 K + 4 V with two Q buffers; BF16 Dqk 128 trades its
  // second Q buffer for a third K stage (S waits on K tiles, P V on V tiles a
  // whole softmax pass later); BF16 Dqk 192 fits 2 + 2 with one Q buffer
  static constexpr int STK = FP8 ? 4 : (DQK == 128 ? 3 : 2);
  static constexpr int STV = FP8 ? 4 : 2;
  static constexpr int QBUF = FP8 ? 2 : 1;           // Q tile buffers (units in flight)
  // K tiles the producer keeps ahead of V.  BF16: the whole K ring, so that
  // loading K(g + STK) waits only for S(g) to finish and never queues behind
  // V(g + 1), whose stage frees a whole softmax pass later (P V(g - 1)).
  static constexpr int KLEAD = FP8 ? STK - STV + 1 : STK;
  static constexpr int NPB = FP8 ? 3 : 2;            // P buffers (tile g uses g % NPB)
  // BF16 Dqk 128: Q in TMEM (A of the S MMAs), one S buffer
  static constexpr bool QTM = !FP8 && DQK == 128;
  static constexpr int NK_QK = ROWB / 32;            // QK MMA K-steps of 32 bytes
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + QBUF * QB;
  static constexpr int OFF_V = OFF_K + STK * KB;
  static constexpr int OFF_ONES = OFF_V + STV * VB;   // FP8: 16 x 128 bytes of e4m3 1.0
  static constexpr int OFF_SF = OFF_ONES + (FP8 ? 2048 : 0);   // FP8: NPB x 512 B scale factors
  // unit hand-over ring: reference max per slot x group x row, and (BF16)
  // the group's partial row sum in a second array of the same shape
  static constexpr int HAND = kHandSlots * 2 * 128 * 4;
  static constexpr int OFF_HAND = OFF_SF + (FP8 ? NPB * 512 : 0);
  static constexpr int OFF_XCH = OFF_HAND + (FP8 ? 1 : 2) * HAND;   // running max per group (2 x 128)
  static constexpr int OFF_BAR = OFF_XCH + 1024;
  // Barriers (phase bookkeeping: every waiter is at most one phase behind,
  // so a parity test cannot alias): Q full/empty per Q buffer; OF = O read
  // by the epilogue (per unit); OFIN = last P V of a unit done (per unit);
  // per S buffer: SF = S full, SC = S read, MX = running max published; per
  // P buffer: PF = P written and O rescaled (ready for P V), PE = P V done (P
  // buffer free, O updated); per hand-over slot: LF = both softmax groups
  // wrote their unit hand-over.
  enum { QF0 = 0, QF1, QE0, QE1, OF, OFIN, DRAIN, DRAIN2, SF0, SF1, SC0, SC1, PF0, PF1, PF2, PE0, PE1, PE2,
         MX0, MX1, LF0, KF = LF0 + kHandSlots };
  static constexpr int KE = KF + STK, VF = KF + 2 * STK, VE = VF + STV;
  static constexpr int NBAR = VE + STV;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;  // + alignment slack
  // tensor-memory columns (512 allocated).  S buffers 0..127 and 128..255 (one
  // S buffer at 0 with Q in TMEM), O 256..383 (128..255 with Q in TMEM), Q
  // 384..447 (bf16 pairs, the A layout of the S MMA)
  static constexpr uint32_t TS0 = 0, TS1 = QTM ? 0 : 128, TO = QTM ? 128 : 256, TQ = 384;
  static constexpr uint32_t TL = 384, TSFB = 400;
  // P buffer b: FP8 32 columns of packed codes at 416 + 32 b; BF16 64 columns
  // of bf16 pairs at 384 + 64 b (256 + 64 b with Q in TMEM); FP8 scale
  // factors of P buffer b at 404 + 4 b
  static __device__ __forceinline__ uint32_t tp(uint32_t b) {
    return FP8 ? 416 + 32 * b : (QTM ? 256 : 384) + 64 * b;
  }
  static __device__ __forceinline__ uint32_t tsfa(uint32_t b) { return 404 + 4 * b; }
  static constexpr uint32_t IDESC_QK = idesc_dense(FP8 ? 0 : 1, FP8 ? 0 : 1, 0, 0, 128, 128);
  static constexpr uint32_t IDESC_PV_BF16 = idesc_dense(1, 1, 0, 1, 128, 128);
  static_assert(SMEM <= 232448, "shared memory budget");
};

#define ZYFA_HD __host__ __device__

ZYFA_HD __forceinline__ int imin(int x, int y) { return x < y ? x : y; }

// Static causal-aware schedule.  Units are grouped by (batch, kv head) slots so
// that one group's K/V stays resident in L2; inside a group the heaviest query
// tiles (most KV tiles) come first, and consecutive units share a kv head.
// Units are dealt round-robin to the persistent CTAs, reversing direction on
// every round so per-CTA work evens out.  Host-callable, so the schedule a
// launch will run can be enumerated on the CPU.
struct UnitIter {
  int G, c, Tq, gq, Hkv, slots, Gk, ngroups;
  int g, k, slots_g, U_g;
  ZYFA_HD void init(int grid, int cta, int Tq_, int Hq, int Hkv_, int B, int Gk_) {
    G = grid; c = cta; Tq = Tq_; Hkv = Hkv_; gq = Hq / Hkv_;
    slots = B * Hkv_; Gk = Gk_; ngroups = (slots + Gk - 1) / Gk;
    g = 0; k = 0;
    slots_g = imin(Gk, slots); U_g = slots_g * gq * Tq;
  }
  // the variable-length signature, so both iterators take the same calls
  ZYFA_HD bool next(int& b, int& hkv, int& hq, int& qt, int& r0, int& len) {
    r0 = 0; len = 0;
    return next(b, hkv, hq, qt);
  }
  ZYFA_HD bool next(int& b, int& hkv, int& hq, int& qt) {
    while (g < ngroups) {
      if (k * G >= U_g) {
        ++g; k = 0;
        if (g < ngroups) { slots_g = imin(Gk, slots - g * Gk); U_g = slots_g * gq * Tq; }
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

// Variable-length batch: sequences packed back to back along the row
// dimension, sequence s holding rows cu[s] .. cu[s+1]-1 of every tensor.  The
// host orders the sequences longest first; a (sequence, kv head) slot is
// s_i * Hkv + hkv for the i-th sequence of that order.  The table travels as
// a kernel parameter (with AttnArgs inside the 4 KiB parameter space).
constexpr int kMaxVarlenSeqs = 384;
struct VarlenSeqs {
  int n;                          // sequences
  int kv_row_bytes;               // bytes of one K row plus one V row of one kv head
  long long group_bytes;          // K/V bytes a scheduling group may hold (L2 budget)
  int order[kMaxVarlenSeqs];      // sequence ids, longest first (equal lengths by id)
  int cu[kMaxVarlenSeqs + 1];     // first packed row of each sequence; cu[n] = total rows
};

// The same schedule over a variable-length batch.  Slots, in the order above,
// are grouped greedily: a group takes slots while their K/V bytes fit the L2
// budget (at least one slot).  Inside a group units are issued by query tile
// index descending (level L = the tile index), a level holding every (slot,
// query head) whose sequence has more than L tiles; slots are longest first,
// so those are a prefix of the group and the prefix only grows as L falls.
// With all lengths equal this is UnitIter's schedule, unit for unit.
struct VarlenIter {
  const VarlenSeqs* t;
  int G, c, gq, Hkv, nslots;
  int s0, s1;          // the group's slots [s0, s1)
  int k, U;            // dealing round; units of the group
  int L, base, act;    // current level, its first unit index, slots active at it
  ZYFA_HD int seq_len(int slot) const {
    const int s = t->order[slot / Hkv];
    return t->cu[s + 1] - t->cu[s];
  }
  ZYFA_HD int tiles(int slot) const { return (seq_len(slot) + 127) / 128; }
  ZYFA_HD void open(int from) {
    s0 = from; s1 = from; U = 0; k = 0;
    long long bytes = 0;
    while (s1 < nslots) {
      const long long sb = static_cast<long long>(seq_len(s1)) * t->kv_row_bytes;
      if (s1 > s0 && bytes + sb > t->group_bytes) break;
      bytes += sb;
      U += tiles(s1);
      ++s1;
    }
    U *= gq;
    L = s0 < nslots ? tiles(s0) - 1 : -1;
    base = 0; act = 0;
    while (s0 + act < s1 && tiles(s0 + act) > L) ++act;
  }
  ZYFA_HD void init(int grid, int cta, const VarlenSeqs* seqs, int Hq, int Hkv_) {
    t = seqs; G = grid; c = cta; Hkv = Hkv_; gq = Hq / Hkv_; nslots = seqs->n * Hkv_;
    open(0);
  }
  ZYFA_HD bool next(int& b, int& hkv, int& hq, int& qt) {
    int r0, len;
    return next(b, hkv, hq, qt, r0, len);
  }
  // b: sequence id; r0, len: its first packed row and its length
  ZYFA_HD bool next(int& b, int& hkv, int& hq, int& qt, int& r0, int& len) {
    while (s0 < nslots) {
      if (k * G >= U) { open(s1); continue; }
      const int p = k * G + ((k & 1) ? (G - 1 - c) : c);
      ++k;
      if (p >= U) continue;
      while (p >= base + act * gq) {   // p < U, so this stops at a level >= 0
        base += act * gq;
        --L;
        while (s0 + act < s1 && tiles(s0 + act) > L) ++act;
      }
      const int rem = p - base, slot = s0 + rem / gq, i = slot / Hkv;
      b = t->order[i];
      hkv = slot - i * Hkv;
      hq = hkv * gq + (rem - (rem / gq) * gq);
      qt = L;
      r0 = t->cu[b];
      len = t->cu[b + 1] - r0;
      return true;
    }
    return false;
  }
};

// One lane of a converged warp (the same lane every time for the same mask).
__device__ __forceinline__ bool elect_one() {
  uint32_t pred;
  asm volatile(
      "{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(pred));
  return pred != 0;
}

// The CTA's sequence of (unit, KV tile) pairs in issue order; g counts tiles
// and u counts units across the whole sequence (ring stages and barrier phases
// derive from them).  KT keys per KV tile (128, or 256 for the wide FP8
// kernel): a unit of query tile qt visits tiles 0 .. qt*128/KT.  VARLEN: r0
// and len are the unit's sequence's first packed row and length.
template <bool VARLEN, int KT = 128>
struct TileStream {
  typename std::conditional<VARLEN, VarlenIter, UnitIter>::type units;
  int b, hkv, hq, qt, j, nkv;
  int r0, len;
  uint32_t g, u;
  __device__ void init(int grid, int cta, const AttnArgs& a, const VarlenSeqs* vs) {
    if constexpr (VARLEN) units.init(grid, cta, vs, a.Hq, a.Hkv);
    else units.init(grid, cta, a.Tq, a.Hq, a.Hkv, a.B, a.group_slots);
    j = 0; nkv = 0; g = 0xffffffffu; u = 0xffffffffu;
    r0 = 0; len = 0;
  }
  __device__ bool next() {
    if (j + 1 < nkv) { ++j; ++g; return true; }
    if constexpr (VARLEN) {
      if (!units.next(b, hkv, hq, qt, r0, len)) return false;
    } else {
      if (!units.next(b, hkv, hq, qt)) return false;
    }
    nkv = qt * 128 / KT + 1; j = 0; ++g; ++u;
    return true;
  }
};

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Two fp32 values -> two e4m3 codes (round to nearest even, saturating), the
// first value's code in the low byte.
__device__ __forceinline__ uint32_t pack_e4m3x2(float lo, float hi) {
  uint16_t d;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(hi), "f"(lo));
  return d;
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

// Max of 64 consecutive fp32 values (held as bits): 3-input max, 4 chains.
__device__ __forceinline__ float max64(const uint32_t* s) {
  float a[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)                       // elements 0 .. 11
    a[i] = max3f(__uint_as_float(s[i]), __uint_as_float(s[4 + i]), __uint_as_float(s[8 + i]));
#pragma unroll
  for (int c = 12; c < 60; c += 8)                  // elements 12 .. 59
#pragma unroll
    for (int i = 0; i < 4; ++i) a[i] = max3f(a[i], __uint_as_float(s[c + i]), __uint_as_float(s[c + 4 + i]));
#pragma unroll
  for (int i = 0; i < 4; ++i) a[i] = fmaxf(a[i], __uint_as_float(s[60 + i]));   // 60 .. 63
  return max3f(fmaxf(a[0], a[1]), a[2], a[3]);
}

// EXACTP (FP8 only): the ablation that writes P the conventional way, an
// exponential (MUFU ex2) followed by a conversion to e4m3, with the same block
// shift, scale factors and row sum as Lean P.
//
// VARLEN: the batch is packed (rows of sequence s at cu[s] .. cu[s+1]-1, one
// tensor-map batch), and vs holds the sequences; otherwise vs is null.
template <bool VARLEN> struct SeqTable {};
template <> struct SeqTable<true> : VarlenSeqs {};
template <bool FP8, int DQK, bool EXACTP = false, bool VARLEN = false>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_fwd_kernel(const __grid_constant__ AttnArgs a, const __grid_constant__ SeqTable<VARLEN> seqs) {
  const VarlenSeqs* vs = nullptr;
  if constexpr (VARLEN) vs = &seqs;
  using Cf = AttnCfg<FP8, DQK>;
  using TS = TileStream<VARLEN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  const uint32_t sb = smem_u32(sm);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  auto bar = [&](int i) -> uint32_t { return sb + Cf::OFF_BAR + 8u * static_cast<uint32_t>(i); };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sm + Cf::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + Cf::OFF_MISC + 4);
  float* hand_m = reinterpret_cast<float*>(sm + Cf::OFF_HAND);               // [slot][group][row]
  float* hand_l = reinterpret_cast<float*>(sm + Cf::OFF_HAND + Cf::HAND);    // BF16 only, same shape
  uint32_t* sf_s = reinterpret_cast<uint32_t*>(sm + Cf::OFF_SF);
  float* xch_s = reinterpret_cast<float*>(sm + Cf::OFF_XCH);

  if (tid == 0) {
    *abort_flag = 0;
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(Cf::QF0 + i), 1);
      mbar_init(bar(Cf::QE0 + i), 1);
    }
    mbar_init(bar(Cf::OF), 128);
    mbar_init(bar(Cf::OFIN), 1);
    mbar_init(bar(Cf::DRAIN), 1);
    mbar_init(bar(Cf::DRAIN2), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(Cf::SF0 + i), 1);
      mbar_init(bar(Cf::SC0 + i), 128);
      mbar_init(bar(Cf::MX0 + i), 128);
    }
    for (int i = 0; i < Cf::NPB; ++i) {
      mbar_init(bar(Cf::PF0 + i), 128);
      mbar_init(bar(Cf::PE0 + i), 1);
    }
    for (int i = 0; i < kHandSlots; ++i) mbar_init(bar(Cf::LF0 + i), 256);
    for (int i = 0; i < Cf::STK; ++i) {
      mbar_init(bar(Cf::KF + i), 1);
      mbar_init(bar(Cf::KE + i), 1);
    }
    for (int i = 0; i < Cf::STV; ++i) {
      mbar_init(bar(Cf::VF + i), 1);
      mbar_init(bar(Cf::VE + i), 1);
    }
    fence_mbar_init();
  }
  if (warp == 12 && lane == 0) {
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
    for (int i = tid; i < 512; i += kAttnThreads) ones[i] = 0x38383838u;   // e4m3 1.0
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_holder;
  const WaitCtl ctl{abort_flag, a.timeout_ns};

  if (warp >= 12) {
   reg_dealloc<kRegControl>();
   // The producer and MMA warps run converged; one elected lane polls the
   // barriers and issues the TMA copies / tcgen05 instructions and the
   // commits, so every operand (descriptors, TMEM addresses, coordinates) is
   // warp-uniform.  Warp 15 has no role.
   const bool leader = elect_one();
   const int leader_lane = __ffs(__ballot_sync(0xffffffffu, leader)) - 1;
   auto wait1 = [&](uint32_t br, uint32_t parity) -> bool {
     bool ok = true;
     if (leader) ok = mbar_wait(br, parity, ctl);
     return __shfl_sync(0xffffffffu, ok ? 1 : 0, leader_lane) != 0;
   };
   if (warp == 12) {
    // ------------------------------------------------------------ producer
    // K runs KLEAD tiles ahead of V, in the order the MMAs consume them.
    const uint64_t pol_q = l2_policy_evict_first();
    const uint64_t pol_kv = l2_policy_evict_last();
    TS ks, vst;
    ks.init(gridDim.x, blockIdx.x, a, vs);
    vst.init(gridDim.x, blockIdx.x, a, vs);
    bool ok = true;
    // the last unit / tile whose Q, K and V copies were armed (-1: none): on an
    // abort, the last armed phase of every buffer is waited for, so no copy
    // lands after the CTA exits
    int last_q = -1, last_k = -1, last_v = -1;
    auto load_rows = [&](uint32_t dst, const CUtensorMap* m, const CUtensorMap* mt, uint32_t br,
                         int h, int row, int bb, uint64_t pol) {
#pragma unroll
      for (int c = 0; c < Cf::NCH; ++c)
        tma_load_4d(dst + c * Cf::CHUNK, m, br, c * (128 / Cf::EL), h, row, bb, pol);
      if (Cf::TAIL) tma_load_4d(dst + Cf::NCH * Cf::CHUNK, mt, br, 128, h, row, bb, pol);
    };
    auto load_k = [&](const TS& t) -> bool {
      // checked builds: the unit's indices and its tile's first row
      range_ok(t.b >= 0 && t.b < a.B && t.hq >= 0 && t.hq < a.Hq && t.hkv >= 0 && t.hkv < a.Hkv && t.j >= 0 &&
                   t.j <= t.qt, kChkUnit);
      range_ok(VARLEN ? (t.qt * 128 < t.len && t.r0 >= 0 && t.r0 + t.len <= a.S) : (t.qt * 128 < a.S), kChkRow);
      // tensor-map row and batch coordinates of the unit's sequence
      const int row0 = VARLEN ? t.r0 : 0, tb = VARLEN ? 0 : t.b;
      if (t.j == 0) {                      // first tile of a unit: its Q tile first
        const uint32_t slot = t.u % Cf::QBUF, n = t.u / Cf::QBUF;
        if (n > 0 && !wait1(bar(Cf::QE0 + slot), (n - 1) & 1)) return false;
        if (leader) {
          mbar_arrive_expect_tx(bar(Cf::QF0 + slot), Cf::QB);
          load_rows(sb + Cf::OFF_Q + slot * Cf::QB, &a.map_q, &a.map_q_tail, bar(Cf::QF0 + slot),
                    t.hq, row0 + t.qt * 128, tb, pol_q);
        }
        last_q = static_cast<int>(t.u);
      }
      const uint32_t st = t.g % Cf::STK, n = t.g / Cf::STK;
      if (n > 0 && !wait1(bar(Cf::KE + st), (n - 1) & 1)) return false;
      if (leader) {
        mbar_arrive_expect_tx(bar(Cf::KF + st), Cf::KB);
        load_rows(sb + Cf::OFF_K + st * Cf::KB, &a.map_k, &a.map_k_tail, bar(Cf::KF + st), t.hkv,
                  row0 + t.j * 128, tb, pol_kv);
      }
      last_k = static_cast<int>(t.g);
      __syncwarp();
      return true;
    };
    auto load_v = [&](const TS& t) -> bool {
      const int row0 = VARLEN ? t.r0 : 0, tb = VARLEN ? 0 : t.b;
      const uint32_t st = t.g % Cf::STV, n = t.g / Cf::STV;
      if (n > 0 && !wait1(bar(Cf::VE + st), (n - 1) & 1)) return false;
      if (leader) {
        mbar_arrive_expect_tx(bar(Cf::VF + st), Cf::VB);
#pragma unroll
        for (int c = 0; c < Cf::VB / Cf::CHUNK; ++c)
          tma_load_4d(sb + Cf::OFF_V + st * Cf::VB + c * Cf::CHUNK, &a.map_v, bar(Cf::VF + st),
                      c * (128 / Cf::EL), t.hkv, row0 + t.j * 128, tb, pol_kv);
      }
      last_v = static_cast<int>(t.g);
      __syncwarp();
      return true;
    };
    for (int i = 0; i < Cf::KLEAD && ok && ks.next(); ++i) ok = load_k(ks);
    while (ok && vst.next()) {
      if (ks.next()) ok = load_k(ks);
      if (ok) ok = load_v(vst);
    }
    if (!ok && leader) {
      // let the copies already in flight land before the CTA exits: each
      // buffer's last armed phase completes when its bytes have arrived
      // buffer i's last armed use is the largest index <= last with index % n == i
      auto drain_ring = [&](int last, int n, int bar0) {
        for (int i = 0; i < n && i <= last; ++i) {
          const int x = last - (((last - i) % n) + n) % n;
          drain_wait(bar(bar0 + i), static_cast<uint32_t>(x / n) & 1u, 100000000ull);
        }
      };
      drain_ring(last_q, Cf::QBUF, Cf::QF0);
      drain_ring(last_k, Cf::STK, Cf::KF);
      drain_ring(last_v, Cf::STV, Cf::VF);
    }
    __syncwarp();
   } else if (warp == 13 || warp == 14) {
    // ------------------------------------------------------------ MMA issuers
    // warp 13: S for tile g is issued as soon as its K tile is loaded and the
    // softmax has read S of tile g-2 (two S buffers; g-1 with Q in TMEM).
    // warp 14: P V of tile g once the softmax has written P (and rescaled O,
    // when it had to).
    TS ts;
    ts.init(gridDim.x, blockIdx.x, a, vs);
    bool ok = true;
    // descriptor bases; per-step descriptors add (byte offset >> 4) to the low word
    const uint64_t dq = smem_desc(sb + Cf::OFF_Q, 16, 1024, kSw128);
    const uint64_t dq_t = smem_desc(sb + Cf::OFF_Q + Cf::NCH * Cf::CHUNK, 16, 512, kSw64);
    const uint64_t dk = smem_desc(sb + Cf::OFF_K, 16, 1024, kSw128);
    const uint64_t dk_t = smem_desc(sb + Cf::OFF_K + Cf::NCH * Cf::CHUNK, 16, 512, kSw64);
    const uint64_t dv = smem_desc(sb + Cf::OFF_V, 16384, 1024, kSw128);
    const uint64_t dones = smem_desc(sb + Cf::OFF_ONES, 16, 1024, kSw128);
    const uint64_t dsf = smem_desc(sb + Cf::OFF_SF, 16, 128, kSwNone);
    auto issue_qk = [&](const TS& t) -> bool {
      const uint32_t slot = t.u % Cf::QBUF;
      if (t.j == 0 && !wait1(bar(Cf::QF0 + slot), (t.u / Cf::QBUF) & 1)) return false;
      const uint32_t st = t.g % Cf::STK, buf = Cf::QTM ? 0 : (t.g & 1);
      if (!wait1(bar(Cf::KF + st), (t.g / Cf::STK) & 1)) return false;
      if (Cf::QTM) {
        // one S buffer: the softmax has read S of the previous tile (so the
        // S MMAs of the previous unit, which read Q from TMEM, are done)
        if (t.g >= 1 && !wait1(bar(Cf::SC0), (t.g - 1) & 1)) return false;
      } else if (t.g >= 2 && !wait1(bar(Cf::SC0 + buf), ((t.g >> 1) - 1) & 1)) {
        return false;
      }
      tc_fence_after();
      const uint64_t dqs = dq + ((slot * Cf::QB) >> 4), dqs_t = dq_t + ((slot * Cf::QB) >> 4);
      const uint64_t dks = dk + ((st * Cf::KB) >> 4), dks_t = dk_t + ((st * Cf::KB) >> 4);
      const uint32_t ts = tbase + (buf ? Cf::TS1 : Cf::TS0);
      if (Cf::QTM && leader) {
        if (t.j == 0) {
          // the unit's Q tile into TMEM, one 128 x 32-byte K slice per copy,
          // in the lane / column layout of an A operand; the copies run
          // before the MMAs issued after them
#pragma unroll
          for (int kk = 0; kk < Cf::NK_QK; ++kk)
            tmem_cp_128x256b(tbase + Cf::TQ + 8 * kk, dqs + (((kk >> 2) * Cf::CHUNK + (kk & 3) * 32) >> 4));
          tc_commit(bar(Cf::QE0 + slot));   // the Q slot in shared memory is free
        }
#pragma unroll
        for (int kk = 0; kk < Cf::NK_QK; ++kk)
          mma_f16_ts(ts, tbase + Cf::TQ + 8 * kk, dks + (((kk >> 2) * Cf::CHUNK + (kk & 3) * 32) >> 4),
                     Cf::IDESC_QK, kk > 0 ? 1u : 0u);
        tc_commit(bar(Cf::SF0));
        tc_commit(bar(Cf::KE + st));
      } else if (leader) {
#pragma unroll
        for (int kk = 0; kk < Cf::NK_QK; ++kk) {
          uint64_t ad, bd;
          if (kk < Cf::NCH * 4) {
            const uint32_t off = ((kk >> 2) * Cf::CHUNK + (kk & 3) * 32) >> 4;
            ad = dqs + off; bd = dks + off;
          } else {
            const uint32_t off = ((kk - Cf::NCH * 4) * 32) >> 4;
            ad = dqs_t + off; bd = dks_t + off;
          }
          if (FP8) mma_f8_ss(ts, ad, bd, Cf::IDESC_QK, kk > 0 ? 1u : 0u);
          else mma_f16_ss(ts, ad, bd, Cf::IDESC_QK, kk > 0 ? 1u : 0u);
        }
        tc_commit(bar(Cf::SF0 + buf));
        tc_commit(bar(Cf::KE + st));
        if (t.j == t.nkv - 1) tc_commit(bar(Cf::QE0 + slot));
      }
      __syncwarp();
      return true;
    };
    auto issue_pv = [&](const TS& t) -> bool {
      const uint32_t st = t.g % Cf::STV, buf = t.g % Cf::NPB, ph = (t.g / Cf::NPB) & 1;
      const bool first = t.j == 0;
      // O is free once the previous unit's epilogue has read it
      if (first && t.u > 0 && !wait1(bar(Cf::OF), (t.u - 1) & 1)) return false;
      if (!wait1(bar(Cf::VF + st), (t.g / Cf::STV) & 1)) return false;
      if (!wait1(bar(Cf::PF0 + buf), ph)) return false;   // P stored, O rescaled
      tc_fence_after();
      const uint64_t dvs = dv + ((st * Cf::VB) >> 4);
      const uint32_t tp = tbase + Cf::tp(buf);
      if (leader) {
        if (FP8) {
          const uint32_t sfa = tbase + Cf::tsfa(buf);
          const uint32_t sfb = tbase + Cf::TSFB;
          // scale factors of P: 32 rows x 16 bytes in shared memory, copied to
          // all four lane quarters (the layout the block-scaled MMA reads)
          tmem_cp_32x128b_warpx4(sfa, dsf + ((buf * 512) >> 4));
#pragma unroll
          for (uint32_t k4 = 0; k4 < 4; ++k4)
            mma_mxf8_ts(tbase + Cf::TO, tp + 8 * k4, dvs + ((k4 * 4096) >> 4), idesc_mxf8(1, 128, 128, k4, k4),
                        sfa | (k4 << 30), sfb | (k4 << 30), (!first || k4 > 0) ? 1u : 0u);
#pragma unroll
          for (uint32_t k4 = 0; k4 < 4; ++k4)
            mma_mxf8_ts(tbase + Cf::TL, tp + 8 * k4, dones + ((k4 * 32) >> 4), idesc_mxf8(0, 128, 16, k4, k4),
                        sfa | (k4 << 30), sfb | (k4 << 30), (!first || k4 > 0) ? 1u : 0u);
        } else {
#pragma unroll
          for (uint32_t k8 = 0; k8 < 8; ++k8)
            mma_f16_ts(tbase + Cf::TO, tp + 8 * k8, dvs + ((k8 * 2048) >> 4), Cf::IDESC_PV_BF16,
                       (!first || k8 > 0) ? 1u : 0u);
        }
        tc_commit(bar(Cf::VE + st));
        tc_commit(bar(Cf::PE0 + buf));    // P (and its scale factors) of this buffer consumed
        if (t.j == t.nkv - 1) tc_commit(bar(Cf::OFIN));
      }
      __syncwarp();
      return true;
    };
    if (warp == 13) {
      while (ok && ts.next()) ok = issue_qk(ts);
    } else {
      while (ok && ts.next()) ok = issue_pv(ts);
    }
    // all MMAs issued by this warp's leader must finish before TMEM is released
    if (leader) {
      const uint32_t dr = bar(warp == 13 ? Cf::DRAIN : Cf::DRAIN2);
      tc_commit(dr);
      drain_wait(dr, 0, 100000000ull);
    }
    __syncwarp();
   }
  } else if (warp < 8) {
    reg_alloc<kRegSoftmax>();
    // ------------------------------------------------------------ softmax warpgroups
    // Two groups alternate over the KV tiles: group x = warp / 4 takes the
    // tiles with (g & 1) == x, i.e. always S buffer x (with Q in TMEM the one
    // S buffer, taken in turns), so one group computes while the other waits
    // for its next S.  Thread t of a group owns row
    // 32 (w % 4) + lane (TMEM lane quarter w % 4) and all 128 keys of its
    // tiles.  The running max crosses between the groups once per tile (smem
    // + per-buffer barrier MX), the only serial dependency.
    const int grp = warp >> 2;
    const int row = 32 * (warp & 3) + lane;   // query row inside the tile == TMEM lane
    const uint32_t lb = tbase + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    bool ok = true;
    if (FP8 && grp == 0) {
      tmem_st4(lb + Cf::TSFB, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu);  // scale 1.0
      tmem_wait_st();
    }
    // scale-factor word of row r: bytes at (r % 32) * 16 + (r / 32) * 4
    const uint32_t sf_row = (row & 31) * 4 + (row >> 5);
    const uint32_t ts = lb + (grp ? Cf::TS1 : Cf::TS0);
    TS t;
    t.init(gridDim.x, blockIdx.x, a, vs);
    float A = a.C;
    // this group's latest reference max in the unit, and (BF16) its partial
    // row sum relative to that max
    float l = 0.0f, m_own = __int_as_float(0xff800000);
    while (ok && t.next()) {
      const uint32_t g = t.g;
      if (t.j == 0) {
        l = 0.0f;
        m_own = __int_as_float(0xff800000);
        if (FP8) {
          const bool sok = range_ok(t.b >= 0 && t.b < a.B && t.hq >= 0 && t.hq < a.Hq && t.hkv >= 0 &&
                                    t.hkv < a.Hkv, kChkScale);
          const float qs = (a.q_scale && sok) ? a.q_scale[t.b * a.Hq + t.hq] : 1.0f;
          const float ks = (a.k_scale && sok) ? a.k_scale[t.b * a.Hkv + t.hkv] : 1.0f;
          A = leanp_slope(qs, ks, a.C);
        }
      }
      if ((g & 1) == static_cast<uint32_t>(grp)) {
        const bool diag = t.j == t.qt;
        // one S buffer: the other group's max of tile g-1, published after
        // it read S of tile g-1, keeps the wait on S at most one phase behind
        if (Cf::QTM && g >= 1 &&
            !(ok = warp_wait(bar(Cf::MX0 + ((g - 1) & 1)), ((g - 1) >> 1) & 1, ctl))) break;
        if (!(ok = warp_wait(bar(Cf::SF0 + (Cf::QTM ? 0 : grp)), Cf::QTM ? (g & 1) : ((g >> 1) & 1), ctl))) break;
        tc_fence_after();
        // the whole 128-key row of S in one TMEM round trip; the S buffer is
        // free for the tile after next right away
        uint32_t r[128];
        tmem_ld64p(ts, &r[0]);
        tmem_ld64p(ts + 64, &r[64]);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(bar(Cf::SC0 + (Cf::QTM ? 0 : grp)));
        if (diag) {
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c > row) r[c] = 0xff800000u;   // -inf: key after the query row
        }
        const float bmx0 = max64(&r[0]), bmx1 = max64(&r[64]);
        // running max of the previous tile, from the other group (every tile
        // waits for it, so the exchange buffers are never reused early)
        float m_prev = __int_as_float(0xff800000);
        if (g >= 1) {
          const uint32_t pb = (g - 1) & 1;
          if (!Cf::QTM && !(ok = warp_wait(bar(Cf::MX0 + pb), ((g - 1) >> 1) & 1, ctl))) break;
          if (t.j > 0) m_prev = xch_s[pb * 128 + row];
        }
        // reference max after this tile (FP8: A carries a factor 8)
        float m, alpha = 1.0f;
        const float tmax = fmaxf(bmx0, bmx1);
        if (t.j == 0) {
          m = tmax;
        } else if (__fmul_rn(tmax - m_prev, A) > (FP8 ? 8.0f * kRescaleLog2 : kRescaleLog2)) {
          alpha = ex2_approx(FP8 ? __fmul_rn(__fmul_rn(m_prev - tmax, A), 0.125f)
                                 : __fmul_rn(m_prev - tmax, A));
          m = tmax;
        } else {
          m = m_prev;
        }
        xch_s[grp * 128 + row] = m;
        mbar_arrive(bar(Cf::MX0 + grp));
        // P V of tile g-NPB has read this P buffer (and its scale factors)
        const uint32_t pbuf = g % Cf::NPB;
        const uint32_t tp = lb + Cf::tp(pbuf);
        if (g >= static_cast<uint32_t>(Cf::NPB) &&
            !(ok = warp_wait(bar(Cf::PE0 + pbuf), ((g / Cf::NPB) - 1) & 1, ctl))) break;
        if (FP8) {
          uint32_t sfw = 0;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint32_t* rh = &r[64 * h];
            const int jb = leanp_block_shift(m, h ? bmx1 : bmx0, A);
            uint32_t p[16];
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
                p[w] = pack_e4m3x2(e0, e1) | (pack_e4m3x2(e2, e3) << 16);
              }
            } else {
              const float Bb = leanp_row_offset(m, A, jb);
              const float a256 = __fmul_rn(A, 0.00390625f), b256 = __fmul_rn(Bb, 0.00390625f);
#pragma unroll
              for (int w = 0; w < 16; ++w) {
                uint32_t w0, w1, w2, w3;
                leanp_code_word2(__uint_as_float(rh[4 * w]), __uint_as_float(rh[4 * w + 1]), a256, b256, w0, w1);
                leanp_code_word2(__uint_as_float(rh[4 * w + 2]), __uint_as_float(rh[4 * w + 3]), a256, b256, w2, w3);
                p[w] = pack4_codes(w0, w1, w2, w3);
              }
            }
            tmem_st16p(tp + 16 * h, p);
            // E8M0 scale code 127 - j for both 32-key MX blocks of this 64-key block
            sfw |= static_cast<uint32_t>((127 - jb) * 0x0101) << (16 * h);
          }
          sf_s[pbuf * 128 + sf_row] = sfw;
          fence_proxy_async_smem();   // the copy to TMEM reads it through the async proxy
        } else {
          const float mc = m * A;
          const uint64_t A2 = f2_pack(A, A), nmc2 = f2_pack(-mc, -mc);
          uint64_t acc2[2] = {0, 0};
#pragma unroll
          for (int c8 = 0; c8 < 8; ++c8) {
            uint32_t pb[8];
#pragma unroll
            for (int w = 0; w < 8; ++w) {
              float x0, x1;
              f2_unpack(fma2_rn(f2_pack(__uint_as_float(r[16 * c8 + 2 * w]), __uint_as_float(r[16 * c8 + 2 * w + 1])),
                                A2, nmc2), x0, x1);
              const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
              acc2[w & 1] = add2_rn(acc2[w & 1], f2_pack(p0, p1));
              pb[w] = pack_bf16x2(p0, p1);
            }
            tmem_st8p(tp + 8 * c8, pb);
          }
          float s0, s1, s2, s3;
          f2_unpack(acc2[0], s0, s1);
          f2_unpack(acc2[1], s2, s3);
          // this group's partial row sum, kept relative to the newest max
          l = l * ex2_approx(__fmul_rn(m_own - m, A)) + ((s0 + s1) + (s2 + s3));
        }
        m_own = m;
        // the reference max moved: O (and the FP8 row sum) still hold tiles
        // 0 .. g-1 against the old one; rescale this warp's rows once P V of
        // tile g-1 has landed (P V of tile g waits for PF below)
        if (__any_sync(0xffffffffu, alpha != 1.0f)) {
          const uint32_t pg = g - 1;
          if (!(ok = warp_wait(bar(Cf::PE0 + pg % Cf::NPB), (pg / Cf::NPB) & 1, ctl))) break;
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
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(Cf::PF0 + pbuf));
      }
      if (t.j == t.nkv - 1) {
        // the unit's last tile (this group's or the other's): hand this
        // group's final (row sum, reference max) over to the epilogue
        const uint32_t hs = t.u % kHandSlots;
        hand_m[(hs * 2 + grp) * 128 + row] = m_own;
        if (!FP8) hand_l[(hs * 2 + grp) * 128 + row] = l;
        mbar_arrive(bar(Cf::LF0 + hs));
      }
    }
  } else {
    reg_dealloc<kRegEpilogue>();
    // ------------------------------------------------------------ epilogue warpgroup
    const int row = 32 * (warp & 3) + lane;
    const uint32_t lb = tbase + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    typename std::conditional<VARLEN, VarlenIter, UnitIter>::type units;
    if constexpr (VARLEN) units.init(gridDim.x, blockIdx.x, vs, a.Hq, a.Hkv);
    else units.init(gridDim.x, blockIdx.x, a.Tq, a.Hq, a.Hkv, a.B, a.group_slots);
    uint32_t kv_it = 0, u_it = 0;
    int b, hkv, hq, qt;
    int r0 = 0, len = 0;   // VARLEN: the unit's sequence's first packed row and length
    bool ok = true;
    while (ok && (VARLEN ? units.next(b, hkv, hq, qt, r0, len) : units.next(b, hkv, hq, qt))) {
      const int nkv = qt + 1;
      kv_it += nkv;
      // ---- O / l (* v_scale) -> bf16, rows past S are not written
      if (!(ok = warp_wait(bar(Cf::OFIN), u_it & 1, ctl))) break;
      const uint32_t hs = u_it % kHandSlots;
      if (!(ok = warp_wait(bar(Cf::LF0 + hs), (u_it / kHandSlots) & 1, ctl))) break;
      tc_fence_after();
      // the group of the unit's last tile holds the final reference max
      const int gl = static_cast<int>((kv_it - 1) & 1);
      const float m_last = hand_m[(hs * 2 + gl) * 128 + row];
      float inv, lse_log2;   // lse_log2: log-sum-exp of the scaled scores, in binades
      const int grow = qt * 128 + row;
      if (FP8) {
        const bool sok = range_ok(b >= 0 && b < a.B && hq >= 0 && hq < a.Hq && hkv >= 0 && hkv < a.Hkv,
                                  kChkScale);
        const float vsc = (a.v_scale && sok) ? a.v_scale[b * a.Hkv + hkv] : 1.0f;
        const float lv = __uint_as_float(tmem_ld1(lb + Cf::TL));
        tmem_wait_ld();
        inv = vsc / lv;
        if (a.lse) {   // weights are 2^((s - m) A / 8) against the final reference m
          const float qs = (a.q_scale && sok) ? a.q_scale[b * a.Hq + hq] : 1.0f;
          const float ks = (a.k_scale && sok) ? a.k_scale[b * a.Hkv + hkv] : 1.0f;
          const float A8 = __fmul_rn(leanp_slope(qs, ks, a.C), 0.125f);
          lse_log2 = __fmaf_rn(m_last, A8, log2f(lv));
        }
      } else {
        // each group's partial row sum is relative to its own latest max
        const int go = gl ^ 1;
        float lt = hand_l[(hs * 2 + gl) * 128 + row];
        if (nkv >= 2)
          lt += hand_l[(hs * 2 + go) * 128 + row] * ex2_approx(__fmul_rn(hand_m[(hs * 2 + go) * 128 + row] - m_last, a.C));
        inv = 1.0f / lt;
        if (a.lse) lse_log2 = __fmaf_rn(m_last, a.C, log2f(lt));
      }
      // output row: (b, grow) of [B, S, Hq, 128], or packed row r0 + grow of
      // [T, Hq, 128]; lse [B, Hq, S] or [Hq, T]
      // checked builds: a row that is stored must lie inside the tensor
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
        tmem_ld32p(lb + Cf::TO + 32 * q, o);
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
      mbar_arrive(bar(Cf::OF));
      ++u_it;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tbase, 512);
}

static_assert(sizeof(AttnArgs) + sizeof(VarlenSeqs) <= 4096, "kernel parameter space");

}  // namespace zyfa

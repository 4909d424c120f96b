// zyfa.cu -- the C ABI of libzyfa.so (declared in include/zyfa.h): argument
// validation, TMA descriptor encoding, instance selection and launches.  All
// device code of the library is in this one translation unit.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <mutex>
#include <utility>
#include <numeric>
#include <vector>

#include "../../include/zyfa.h"
#include "attn_fwd.cuh"
#include "attn_fwd_wide.cuh"
#include "leanp.cuh"
#include "ptx.cuh"
#include "quantize.cuh"

namespace zyfa {

// ---------------------------------------------------------------- helpers

constexpr int kMaxDevices = 64;
constexpr unsigned long long kDefaultTimeoutNs = 2000000000ull;

std::atomic<unsigned long long> g_timeout_ns{0};

unsigned long long wait_timeout_ns() {
  unsigned long long t = g_timeout_ns.load(std::memory_order_relaxed);
  if (t != 0) return t;
  t = kDefaultTimeoutNs;
  if (const char* e = std::getenv("ZYFA_WAIT_TIMEOUT_MS")) {
    const double ms = std::atof(e);
    if (ms > 0) t = static_cast<unsigned long long>(ms * 1e6);
  }
  g_timeout_ns.store(t, std::memory_order_relaxed);
  return t;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

struct DeviceInfo {
  int sms = 0;
  bool attr_set[14] = {};
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

// 4-D map over a BSHD tensor: dims (D, H, S, B) innermost first; a box is
// `box_d` elements of one head for 128 consecutive sequence rows.  Rows past S
// read as zero.
bool make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int el, int B, int S, int H,
              int D, int box_d, CUtensorMapSwizzle swz) {
  const EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)S, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)D * el, (cuuint64_t)H * D * el, (cuuint64_t)S * H * D * el};
  cuuint32_t box[4] = {(cuuint32_t)box_d, 1, 128, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, dt, 4, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// K/V bytes one scheduling group may hold: its tiles stay resident in L2
// (126 MB on B200) while the group's query tiles stream through.
constexpr long long kGroupBytes = 48ll * 1024 * 1024;

// (batch, kv head) slots per scheduling group of a fixed-length launch
int group_slots_for(int B, int Hkv, int S, int dqk, int el) {
  const double kv_slot_bytes = static_cast<double>(S) * (dqk + 128) * el;
  long long gk = static_cast<long long>(static_cast<double>(kGroupBytes) / kv_slot_bytes);
  const long long slots = static_cast<long long>(B) * Hkv;
  if (gk < 1) gk = 1;
  if (gk > slots) gk = slots;
  return static_cast<int>(gk);
}

// The sequence table of a variable-length launch: ids ordered longest first
// (a stable sort, so equal lengths keep their order), offsets as given.
void fill_varlen_table(VarlenSeqs& t, const int* cu, int nseq, int dqk, int el) {
  t.n = nseq;
  t.kv_row_bytes = (dqk + 128) * el;
  t.group_bytes = kGroupBytes;
  for (int i = 0; i <= nseq; ++i) t.cu[i] = cu[i];
  std::vector<int> ids(nseq);
  std::iota(ids.begin(), ids.end(), 0);
  std::stable_sort(ids.begin(), ids.end(),
                   [&](int x, int y) { return cu[x + 1] - cu[x] > cu[y + 1] - cu[y]; });
  for (int i = 0; i < nseq; ++i) t.order[i] = ids[i];
}

long long varlen_units(const int* cu, int nseq, int Hq) {
  long long u = 0;
  for (int i = 0; i < nseq; ++i) u += static_cast<long long>(Hq) * ((cu[i + 1] - cu[i] + 127) / 128);
  return u;
}

// Tensor maps and scalar arguments shared by both launch forms.  B, S are the
// tensor-map batch and row extents (a packed batch: 1, total rows).
template <bool FP8, int DQK>
bool fill_attn_args(AttnArgs& a, const void* q, const void* k, const void* v, void* o, int B, int Hq, int Hkv,
                    int S, const float* qs, const float* ks, const float* vs, float* lse) {
  using Cf = AttnCfg<FP8, DQK>;
  const CUtensorMapDataType dt = FP8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const int el = FP8 ? 1 : 2;
  const int box = 128 / el;   // 128 bytes of one row
  bool ok = make_map(&a.map_q, q, dt, el, B, S, Hq, DQK, box, CU_TENSOR_MAP_SWIZZLE_128B) &&
            make_map(&a.map_k, k, dt, el, B, S, Hkv, DQK, box, CU_TENSOR_MAP_SWIZZLE_128B) &&
            make_map(&a.map_v, v, dt, el, B, S, Hkv, 128, box, CU_TENSOR_MAP_SWIZZLE_128B);
  if (Cf::TAIL) {
    ok = ok && make_map(&a.map_q_tail, q, dt, el, B, S, Hq, DQK, 64, CU_TENSOR_MAP_SWIZZLE_64B) &&
         make_map(&a.map_k_tail, k, dt, el, B, S, Hkv, DQK, 64, CU_TENSOR_MAP_SWIZZLE_64B);
  } else {
    a.map_q_tail = a.map_q;
    a.map_k_tail = a.map_k;
  }
  if (!ok) return false;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  a.q_scale = qs;
  a.k_scale = ks;
  a.v_scale = vs;
  a.Hq = Hq; a.Hkv = Hkv;
  a.C = FP8 ? static_cast<float>(8.0 * 1.4426950408889634074 / std::sqrt(static_cast<double>(DQK)))
            : static_cast<float>(1.4426950408889634074 / std::sqrt(static_cast<double>(DQK)));
  a.timeout_ns = wait_timeout_ns();
  return true;
}

// SM count of the device, and a kernel instance's shared-memory opt-in (once)
template <typename Kernel>
bool prepare_kernel(int dev, int inst, Kernel kernel, int smem) {
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo& di = g_dev[dev];
  if (di.sms == 0 && cudaDeviceGetAttribute(&di.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return false;
  if (!di.attr_set[inst]) {
    // the warpgroups' setmaxnreg shares must add up to what the launch holds:
    // a raise asking for more than that would wait forever, so a build whose
    // register count differs is refused here, before any launch
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kernel) != cudaSuccess || fa.numRegs != kLaunchRegs) return false;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return false;
    di.attr_set[inst] = true;
  }
  return true;
}

template <bool FP8, int DQK, bool EXACTP, bool VARLEN>
bool prepare_device(int dev, int inst) {
  return prepare_kernel(dev, inst, attn_fwd_kernel<FP8, DQK, EXACTP, VARLEN>, AttnCfg<FP8, DQK>::SMEM);
}

template <bool FP8, int DQK, bool EXACTP = false>
int launch_attn(const void* q, const void* k, const void* v, void* o, int B, int Hq, int Hkv, int S,
                const float* qs, const float* ks, const float* vs, cudaStream_t stream, int dev,
                int inst, float* lse = nullptr) {
  using Cf = AttnCfg<FP8, DQK>;
  AttnArgs a;
  if (!fill_attn_args<FP8, DQK>(a, q, k, v, o, B, Hq, Hkv, S, qs, ks, vs, lse)) return ZYFA_ERR_CUDA;
  a.B = B; a.S = S;
  a.Tq = (S + 127) / 128;
  a.group_slots = group_slots_for(B, Hkv, S, DQK, FP8 ? 1 : 2);
  if (!prepare_device<FP8, DQK, EXACTP, false>(dev, inst)) return ZYFA_ERR_CUDA;
  const long long units = static_cast<long long>(B) * Hq * a.Tq;
  const int grid = static_cast<int>(units < g_dev[dev].sms ? units : g_dev[dev].sms);
  attn_fwd_kernel<FP8, DQK, EXACTP><<<grid, kAttnThreads, Cf::SMEM, stream>>>(a, SeqTable<false>{});
  return cudaGetLastError() == cudaSuccess ? ZYFA_OK : ZYFA_ERR_CUDA;
}

// Variable-length batch: q/k/v/o packed [T, H, D] with T = cu[nseq].
template <bool FP8, int DQK>
int launch_attn_varlen(const void* q, const void* k, const void* v, void* o, const int* cu, int nseq, int Hq,
                       int Hkv, const float* qs, const float* ks, const float* vs, cudaStream_t stream, int dev,
                       int inst, float* lse) {
  using Cf = AttnCfg<FP8, DQK>;
  const long long units = varlen_units(cu, nseq, Hq);
  if (units == 0) return ZYFA_OK;   // every sequence empty: nothing to write
  const int T = cu[nseq];
  AttnArgs a;
  if (!fill_attn_args<FP8, DQK>(a, q, k, v, o, 1, Hq, Hkv, T, qs, ks, vs, lse)) return ZYFA_ERR_CUDA;
  a.B = nseq; a.S = T;
  a.Tq = 0; a.group_slots = 0;   // the sequence table drives the schedule
  SeqTable<true> t;
  fill_varlen_table(t, cu, nseq, DQK, FP8 ? 1 : 2);
  if (!prepare_device<FP8, DQK, false, true>(dev, inst)) return ZYFA_ERR_CUDA;
  const int grid = static_cast<int>(units < g_dev[dev].sms ? units : g_dev[dev].sms);
  attn_fwd_kernel<FP8, DQK, false, true><<<grid, kAttnThreads, Cf::SMEM, stream>>>(a, t);
  return cudaGetLastError() == cudaSuccess ? ZYFA_OK : ZYFA_ERR_CUDA;
}

// FP8 with Dqk = 128 runs the 256-key-tile kernel (attn_fwd_wide.cuh).
template <bool EXACTP>
int launch_attn_wide(const void* q, const void* k, const void* v, void* o, int B, int Hq, int Hkv, int S,
                     const float* qs, const float* ks, const float* vs, cudaStream_t stream, int dev, int inst,
                     float* lse = nullptr) {
  AttnArgs a;
  if (!fill_attn_args<true, 128>(a, q, k, v, o, B, Hq, Hkv, S, qs, ks, vs, lse)) return ZYFA_ERR_CUDA;
  a.B = B; a.S = S;
  a.Tq = (S + 127) / 128;
  a.group_slots = group_slots_for(B, Hkv, S, 128, 1);
  if (!prepare_kernel(dev, inst, attn_fwd_wide_kernel<EXACTP, false>, WideCfg::SMEM)) return ZYFA_ERR_CUDA;
  const long long units = static_cast<long long>(B) * Hq * a.Tq;
  const int grid = static_cast<int>(units < g_dev[dev].sms ? units : g_dev[dev].sms);
  attn_fwd_wide_kernel<EXACTP, false><<<grid, kAttnThreads, WideCfg::SMEM, stream>>>(a, SeqTable<false>{});
  return cudaGetLastError() == cudaSuccess ? ZYFA_OK : ZYFA_ERR_CUDA;
}

int launch_attn_wide_varlen(const void* q, const void* k, const void* v, void* o, const int* cu, int nseq, int Hq,
                            int Hkv, const float* qs, const float* ks, const float* vs, cudaStream_t stream,
                            int dev, int inst, float* lse) {
  const long long units = varlen_units(cu, nseq, Hq);
  if (units == 0) return ZYFA_OK;
  const int T = cu[nseq];
  AttnArgs a;
  if (!fill_attn_args<true, 128>(a, q, k, v, o, 1, Hq, Hkv, T, qs, ks, vs, lse)) return ZYFA_ERR_CUDA;
  a.B = nseq; a.S = T;
  a.Tq = 0; a.group_slots = 0;
  SeqTable<true> t;
  fill_varlen_table(t, cu, nseq, 128, 1);
  if (!prepare_kernel(dev, inst, attn_fwd_wide_kernel<false, true>, WideCfg::SMEM)) return ZYFA_ERR_CUDA;
  const int grid = static_cast<int>(units < g_dev[dev].sms ? units : g_dev[dev].sms);
  attn_fwd_wide_kernel<false, true><<<grid, kAttnThreads, WideCfg::SMEM, stream>>>(a, t);
  return cudaGetLastError() == cudaSuccess ? ZYFA_OK : ZYFA_ERR_CUDA;
}

// The divisors the prepass kernels need per 16-byte vector, as multipliers.
void set_div_magic(QuantArgs& t, int in_dtype) {
  t.mg_vph = div_magic(static_cast<uint32_t>(t.D / (in_dtype == ZYFA_BF16 ? 8 : 4)));
  t.mg_h = div_magic(static_cast<uint32_t>(t.H));
}

// Launch `kernel` with programmatic stream serialization: it may start while
// the stream's previous kernel runs, and waits for that kernel's results in
// griddep_wait (the prepass kernels after the first one).
template <typename... P, typename... A>
cudaError_t launch_dependent(void (*kernel)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                             A&&... args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<A>(args)...);
}

// Sequence rows per prepass CTA: at most 2^30 elements of one batch entry
// (the kernels count a chunk's rows and 16-byte vectors in 32 bits).
long long prepass_rows(long long rows, int H, int D) {
  const long long cap = std::max(1ll, (1ll << 30) / (static_cast<long long>(H) * D));
  return std::max(1ll, std::min(rows, cap));
}

// ---------------------------------------------------------------- test kernels

// Groups of four elements (i .. i + 3) take the attention kernels' own steps:
// leanp_word2 on two pairs, then pack4_codes; each code is read back from its
// byte of the packed word (a ragged last group repeats its last element).
__global__ void leanp_codes_kernel(const float* s, const float* m, const float* bmax, const float* A,
                                   const unsigned char* masked, int n, unsigned char* code, int* jout) {
  const long long nquads = (static_cast<long long>(n) + 3) / 4;
  for (long long qi = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; qi < nquads;
       qi += static_cast<long long>(gridDim.x) * blockDim.x) {
    float a256[4], b256[4], sv[4];
    int jj[4], idx[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int i = static_cast<int>(4 * qi + e < n ? 4 * qi + e : n - 1);
      idx[e] = i;
      const float Ai = A[i], mi = m[i];
      jj[e] = leanp_block_shift(mi, bmax[i], Ai);
      const float B = leanp_row_offset(mi, Ai, jj[e]);
      sv[e] = (masked && masked[i]) ? __int_as_float(0xff800000) : s[i];
      a256[e] = __fmul_rn(Ai, 0.00390625f);
      b256[e] = __fmul_rn(B, 0.00390625f);
    }
    uint32_t w[4];
    leanp_word2(leanp_scaled_u(sv[0], a256[0], b256[0]), leanp_scaled_u(sv[1], a256[1], b256[1]), w[0], w[1]);
    leanp_word2(leanp_scaled_u(sv[2], a256[2], b256[2]), leanp_scaled_u(sv[3], a256[3], b256[3]), w[2], w[3]);
    const uint32_t packed = pack4_codes(w[0], w[1], w[2], w[3]);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (4 * qi + e >= n) break;
      code[idx[e]] = static_cast<unsigned char>((packed >> (8 * e)) & 0xffu);
      if (jout) jout[idx[e]] = jj[e];
    }
  }
}

__global__ void selftest_wait_kernel(unsigned long long timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
    const WaitCtl ctl{&abort_flag, timeout_ns};
    (void)mbar_wait(smem_u32(&bar), 0, ctl);   // nothing arrives: runs out, records the status
  }
}

}  // namespace zyfa

using namespace zyfa;

// ---------------------------------------------------------------- C ABI

extern "C" const char* zyfa_status_string(int status) {
  switch (status) {
    case ZYFA_OK: return "ok";
    case ZYFA_ERR_NULL_PTR: return "a required pointer is NULL";
    case ZYFA_ERR_BAD_SHAPE: return "bad shape (B, S and head counts must be >= 1 and fit the index range)";
    case ZYFA_ERR_UNSUPPORTED_HEADDIM: return "unsupported head dimension";
    case ZYFA_ERR_BAD_GQA: return "Hq must be a multiple of Hkv";
    case ZYFA_ERR_MISALIGNED: return "misaligned pointer (tensors need 16-byte, scales 4-byte alignment)";
    case ZYFA_ERR_BAD_DTYPE: return "unsupported dtype or flag";
    case ZYFA_ERR_CUDA: return "CUDA call or kernel launch failed";
    case ZYFA_ERR_DEVICE_TIMEOUT: return "a bounded wait inside a kernel ran out";
    default: return "unknown status";
  }
}

extern "C" void zyfa_set_wait_timeout_ns(unsigned long long ns) {
  g_timeout_ns.store(ns, std::memory_order_relaxed);
}

static int attn_validate(const void* q, const void* k, const void* v, void* o, int B, int Hq, int Hkv, int S,
                         int Dqk, int Dv, int dtype, const float* q_scale, const float* k_scale,
                         const float* v_scale) {
  if (!q || !k || !v || !o) return ZYFA_ERR_NULL_PTR;
  if (B < 1 || S < 1 || Hq < 1 || Hkv < 1) return ZYFA_ERR_BAD_SHAPE;
  if (Hq % Hkv != 0) return ZYFA_ERR_BAD_GQA;
  if (!((Dqk == 128 || Dqk == 192) && Dv == 128)) return ZYFA_ERR_UNSUPPORTED_HEADDIM;
  if (dtype != ZYFA_BF16 && dtype != ZYFA_FP8_E4M3) return ZYFA_ERR_BAD_DTYPE;
  // TMA coordinates are 32-bit; the flat element count must fit comfortably
  const long long tq = (static_cast<long long>(S) + 127) / 128;
  if (static_cast<long long>(B) * Hq * tq > (1ll << 31) - 1) return ZYFA_ERR_BAD_SHAPE;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16)) return ZYFA_ERR_MISALIGNED;
  if (dtype == ZYFA_FP8_E4M3 &&
      (!aligned(q_scale, 4) || !aligned(k_scale, 4) || !aligned(v_scale, 4)))
    return ZYFA_ERR_MISALIGNED;
  return ZYFA_OK;
}

extern "C" int zyfa_attn_fwd(const void* q, const void* k, const void* v, void* o, int B, int Hq,
                             int Hkv, int S, int Dqk, int Dv, int dtype, const float* q_scale,
                             const float* k_scale, const float* v_scale, void* stream) {
  const int bad = attn_validate(q, k, v, o, B, Hq, Hkv, S, Dqk, Dv, dtype, q_scale, k_scale, v_scale);
  if (bad != ZYFA_OK) return bad;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ZYFA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == ZYFA_FP8_E4M3) {
    if (Dqk == 128) return launch_attn_wide<false>(q, k, v, o, B, Hq, Hkv, S, q_scale, k_scale, v_scale, st, dev, 10);
    return launch_attn<true, 192>(q, k, v, o, B, Hq, Hkv, S, q_scale, k_scale, v_scale, st, dev, 1);
  }
  if (Dqk == 128) return launch_attn<false, 128>(q, k, v, o, B, Hq, Hkv, S, nullptr, nullptr, nullptr, st, dev, 2);
  return launch_attn<false, 192>(q, k, v, o, B, Hq, Hkv, S, nullptr, nullptr, nullptr, st, dev, 3);
}

extern "C" int zyfa_attn_fwd_lse(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                                 int Hq, int Hkv, int S, int Dqk, int Dv, int dtype, const float* q_scale,
                                 const float* k_scale, const float* v_scale, void* stream) {
  const int bad = attn_validate(q, k, v, o, B, Hq, Hkv, S, Dqk, Dv, dtype, q_scale, k_scale, v_scale);
  if (bad != ZYFA_OK) return bad;
  if (!lse) return ZYFA_ERR_NULL_PTR;
  if (!aligned(lse, 4)) return ZYFA_ERR_MISALIGNED;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ZYFA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == ZYFA_FP8_E4M3) {
    if (Dqk == 128) return launch_attn_wide<false>(q, k, v, o, B, Hq, Hkv, S, q_scale, k_scale, v_scale, st, dev, 10, lse);
    return launch_attn<true, 192>(q, k, v, o, B, Hq, Hkv, S, q_scale, k_scale, v_scale, st, dev, 1, lse);
  }
  if (Dqk == 128) return launch_attn<false, 128>(q, k, v, o, B, Hq, Hkv, S, nullptr, nullptr, nullptr, st, dev, 2, lse);
  return launch_attn<false, 192>(q, k, v, o, B, Hq, Hkv, S, nullptr, nullptr, nullptr, st, dev, 3, lse);
}

extern "C" int zyfa_attn_fwd_fp8_exact_p(const void* q, const void* k, const void* v, void* o, int B, int Hq,
                                         int Hkv, int S, int Dqk, int Dv, const float* q_scale,
                                         const float* k_scale, const float* v_scale, void* stream) {
  const int bad = attn_validate(q, k, v, o, B, Hq, Hkv, S, Dqk, Dv, ZYFA_FP8_E4M3, q_scale, k_scale, v_scale);
  if (bad != ZYFA_OK) return bad;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ZYFA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (Dqk == 128) return launch_attn_wide<true>(q, k, v, o, B, Hq, Hkv, S, q_scale, k_scale, v_scale, st, dev, 11);
  return launch_attn<true, 192, true>(q, k, v, o, B, Hq, Hkv, S, q_scale, k_scale, v_scale, st, dev, 5);
}

extern "C" int zyfa_quantize(const void* x, int in_dtype, void* x_fp8, float* scale, int B, int S, int H,
                             int D, int hadamard, void* stream) {
  if (!x || !x_fp8 || !scale) return ZYFA_ERR_NULL_PTR;
  if (B < 1 || S < 1 || H < 1 || B > 65535 || H > 4096) return ZYFA_ERR_BAD_SHAPE;
  if (in_dtype != ZYFA_BF16 && in_dtype != ZYFA_FP32) return ZYFA_ERR_BAD_DTYPE;
  if (hadamard != 0 && hadamard != 1) return ZYFA_ERR_BAD_DTYPE;
  if (D < 8 || D > 1024 || D % 8 != 0 || (hadamard && D != 128 && D != 192)) return ZYFA_ERR_UNSUPPORTED_HEADDIM;
  if (!aligned(x, 16) || !aligned(x_fp8, 16) || !aligned(scale, 4)) return ZYFA_ERR_MISALIGNED;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess) return ZYFA_ERR_CUDA;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return ZYFA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const long long want = 4ll * sms;
  long long chunks = (want + B - 1) / B;
  if (chunks > S) chunks = S;
  if (chunks < 1) chunks = 1;
  QuantArgs a;
  a.x = x;
  a.out = static_cast<uint8_t*>(x_fp8);
  a.scale = scale;
  a.S = S; a.H = H; a.D = D;
  a.rows_per_cta = static_cast<int>(prepass_rows((S + chunks - 1) / chunks, H, D));
  set_div_magic(a, in_dtype);
  const dim3 grid(static_cast<unsigned>((S + a.rows_per_cta - 1) / a.rows_per_cta), static_cast<unsigned>(B));
  const size_t shm = static_cast<size_t>(H) * 8;   // amax, or scale and its reciprocal, per head
  if (cudaMemsetAsync(scale, 0, static_cast<size_t>(B) * H * sizeof(float), st) != cudaSuccess)
    return ZYFA_ERR_CUDA;
  // the amax pass follows the memset in plain stream order; the codes and
  // finalize passes are dependent launches
  auto run = [&](auto amax_k, auto codes_k) -> cudaError_t {
    amax_k<<<grid, kQuantThreads, shm, st>>>(a);
    const cudaError_t e = cudaGetLastError();
    return e != cudaSuccess ? e : launch_dependent(codes_k, grid, dim3(kQuantThreads), shm, st, a);
  };
  cudaError_t e;
  if (in_dtype == ZYFA_BF16)
    e = hadamard ? run(quant_amax_kernel<__nv_bfloat16, true>, quant_codes_kernel<__nv_bfloat16, true>)
                 : run(quant_amax_kernel<__nv_bfloat16, false>, quant_codes_kernel<__nv_bfloat16, false>);
  else
    e = hadamard ? run(quant_amax_kernel<float, true>, quant_codes_kernel<float, true>)
                 : run(quant_amax_kernel<float, false>, quant_codes_kernel<float, false>);
  if (e != cudaSuccess) return ZYFA_ERR_CUDA;
  const int n = B * H;
  if (launch_dependent(quant_finalize_kernel, dim3((n + 255) / 256), dim3(256), 0, st, scale, n) != cudaSuccess)
    return ZYFA_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? ZYFA_OK : ZYFA_ERR_CUDA;
}

extern "C" int zyfa_quantize_qkv(const void* q, const void* k, const void* v, int in_dtype, void* q_fp8,
                                 void* k_fp8, void* v_fp8, float* q_scale, float* k_scale, float* v_scale,
                                 int B, int S, int Hq, int Hkv, int Dqk, int Dv, int hadamard_qk, void* stream) {
  if (!q || !k || !v || !q_fp8 || !k_fp8 || !v_fp8 || !q_scale || !k_scale || !v_scale) return ZYFA_ERR_NULL_PTR;
  if (B < 1 || S < 1 || Hq < 1 || Hkv < 1 || B > 65535 || Hq > 4096 || Hkv > 4096) return ZYFA_ERR_BAD_SHAPE;
  if (in_dtype != ZYFA_BF16 && in_dtype != ZYFA_FP32) return ZYFA_ERR_BAD_DTYPE;
  if (hadamard_qk != 0 && hadamard_qk != 1) return ZYFA_ERR_BAD_DTYPE;
  for (int d : {Dqk, Dv})
    if (d < 8 || d > 1024 || d % 8 != 0) return ZYFA_ERR_UNSUPPORTED_HEADDIM;
  if (hadamard_qk && Dqk != 128 && Dqk != 192) return ZYFA_ERR_UNSUPPORTED_HEADDIM;
  for (const void* t : {q, k, v, static_cast<const void*>(q_fp8), static_cast<const void*>(k_fp8),
                        static_cast<const void*>(v_fp8)})
    if (!aligned(t, 16)) return ZYFA_ERR_MISALIGNED;
  if (!aligned(q_scale, 4) || !aligned(k_scale, 4) || !aligned(v_scale, 4)) return ZYFA_ERR_MISALIGNED;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess) return ZYFA_ERR_CUDA;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return ZYFA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Quant3Args a;
  const void* xs[3] = {q, k, v};
  void* outs[3] = {q_fp8, k_fp8, v_fp8};
  float* scs[3] = {q_scale, k_scale, v_scale};
  const int Hs[3] = {Hq, Hkv, Hkv}, Ds[3] = {Dqk, Dqk, Dv};
  // CTAs per batch entry, split among the tensors in proportion to their bytes
  // (the rotated path does more work per byte: twice as many CTAs)
  const double want = static_cast<double>(((hadamard_qk ? 8ll : 4ll) * sms + B - 1) / B);
  double bytes[3], total = 0.0;
  for (int i = 0; i < 3; ++i) { bytes[i] = static_cast<double>(Hs[i]) * Ds[i]; total += bytes[i]; }
  a.first[0] = 0;
  int max_h = 1;
  for (int i = 0; i < 3; ++i) {
    long long chunks = static_cast<long long>(want * bytes[i] / total + 0.5);
    if (chunks < 1) chunks = 1;
    if (chunks > S) chunks = S;
    QuantArgs& t = a.t[i];
    t.x = xs[i];
    t.out = static_cast<uint8_t*>(outs[i]);
    t.scale = scs[i];
    t.S = S; t.H = Hs[i]; t.D = Ds[i];
    t.rows_per_cta = static_cast<int>(prepass_rows((S + chunks - 1) / chunks, Hs[i], Ds[i]));
    set_div_magic(t, in_dtype);
    a.had[i] = (i < 2) ? hadamard_qk : 0;
    const long long cols = a.first[i] + (static_cast<long long>(S) + t.rows_per_cta - 1) / t.rows_per_cta;
    if (cols > 0x7fffffffll) return ZYFA_ERR_BAD_SHAPE;
    a.first[i + 1] = static_cast<int>(cols);
    if (Hs[i] > max_h) max_h = Hs[i];
  }
  const dim3 grid(static_cast<unsigned>(a.first[3]), static_cast<unsigned>(B));
  const size_t shm = static_cast<size_t>(max_h) * 8;   // amax, or scale and its reciprocal, per head
  const int n0 = B * Hq, n1 = B * Hkv, n2 = B * Hkv, n = n0 + n1 + n2;
  // the zero step in plain stream order, the other three as dependent launches
  quant3_zero_kernel<<<(n + 255) / 256, 256, 0, st>>>(q_scale, k_scale, v_scale, n0, n1, n2);
  if (cudaGetLastError() != cudaSuccess) return ZYFA_ERR_CUDA;
  const dim3 blk(kQuantThreads);
  cudaError_t e;
  if (in_dtype == ZYFA_BF16) {
    e = launch_dependent(quant3_amax_kernel<__nv_bfloat16>, grid, blk, shm, st, a);
    if (e == cudaSuccess) e = launch_dependent(quant3_codes_kernel<__nv_bfloat16>, grid, blk, shm, st, a);
  } else {
    e = launch_dependent(quant3_amax_kernel<float>, grid, blk, shm, st, a);
    if (e == cudaSuccess) e = launch_dependent(quant3_codes_kernel<float>, grid, blk, shm, st, a);
  }
  if (e == cudaSuccess)
    e = launch_dependent(quant3_finalize_kernel, dim3((n + 255) / 256), dim3(256), 0, st, q_scale, k_scale,
                         v_scale, n0, n1, n2);
  if (e != cudaSuccess) return ZYFA_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? ZYFA_OK : ZYFA_ERR_CUDA;
}

// ---------------------------------------------------------------- variable-length batches

// cu: host array of nseq + 1 packed-row offsets, cu[0] = 0, non-decreasing
static int cu_validate(const int* cu, int nseq, int max_seqs) {
  if (!cu) return ZYFA_ERR_NULL_PTR;
  if (nseq < 1 || nseq > max_seqs) return ZYFA_ERR_BAD_SHAPE;
  if (cu[0] != 0) return ZYFA_ERR_BAD_SHAPE;
  for (int i = 0; i < nseq; ++i)
    if (cu[i + 1] < cu[i]) return ZYFA_ERR_BAD_SHAPE;
  return ZYFA_OK;
}

extern "C" int zyfa_attn_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                                    const int* cu_seqlens, int nseq, int Hq, int Hkv, int Dqk, int Dv, int dtype,
                                    const float* q_scale, const float* k_scale, const float* v_scale,
                                    void* stream) {
  const int badc = cu_validate(cu_seqlens, nseq, kMaxVarlenSeqs);
  if (badc != ZYFA_OK) return badc;
  const int T = cu_seqlens[nseq];
  if (T == 0) {   // every sequence empty: tensors may be NULL, nothing is launched
    if (Hq < 1 || Hkv < 1) return ZYFA_ERR_BAD_SHAPE;
    if (Hq % Hkv != 0) return ZYFA_ERR_BAD_GQA;
    if (!((Dqk == 128 || Dqk == 192) && Dv == 128)) return ZYFA_ERR_UNSUPPORTED_HEADDIM;
    if (dtype != ZYFA_BF16 && dtype != ZYFA_FP8_E4M3) return ZYFA_ERR_BAD_DTYPE;
    return ZYFA_OK;
  }
  // the checks of the fixed-length form, on one batch of T rows
  const int bad = attn_validate(q, k, v, o, 1, Hq, Hkv, T, Dqk, Dv, dtype, q_scale, k_scale, v_scale);
  if (bad != ZYFA_OK) return bad;
  const long long units = varlen_units(cu_seqlens, nseq, Hq);
  if (units > (1ll << 31) - 1) return ZYFA_ERR_BAD_SHAPE;
  if (lse && !aligned(lse, 4)) return ZYFA_ERR_MISALIGNED;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return ZYFA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == ZYFA_FP8_E4M3) {
    if (Dqk == 128)
      return launch_attn_wide_varlen(q, k, v, o, cu_seqlens, nseq, Hq, Hkv, q_scale, k_scale, v_scale, st, dev, 12,
                                     lse);
    return launch_attn_varlen<true, 192>(q, k, v, o, cu_seqlens, nseq, Hq, Hkv, q_scale, k_scale, v_scale, st,
                                         dev, 7, lse);
  }
  if (Dqk == 128)
    return launch_attn_varlen<false, 128>(q, k, v, o, cu_seqlens, nseq, Hq, Hkv, nullptr, nullptr, nullptr, st,
                                          dev, 8, lse);
  return launch_attn_varlen<false, 192>(q, k, v, o, cu_seqlens, nseq, Hq, Hkv, nullptr, nullptr, nullptr, st,
                                        dev, 9, lse);
}

// The prepass over a packed batch for n (1 or 3) tensors sharing cu.
static int quantize_varlen_n(int n, const void* const* xs, void* const* outs, float* const* scs, const int* Hs,
                             const int* Ds, const int* had, int in_dtype, const int* cu, int nseq, void* stream) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess) return ZYFA_ERR_CUDA;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return ZYFA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int T = cu[nseq];
  // CTAs per average sequence as in the fixed-length prepass, split among
  // the tensors in proportion to their bytes; a longer sequence gets
  // proportionally more chunks of the same height
  const long long mean_len = std::max(1ll, (static_cast<long long>(T) + nseq - 1) / nseq);
  bool any_had = false;
  double bytes[3] = {0.0, 0.0, 0.0}, total = 0.0;
  for (int i = 0; i < n; ++i) {
    bytes[i] = static_cast<double>(Hs[i]) * Ds[i];
    total += bytes[i];
    any_had = any_had || had[i];
  }
  const double want = static_cast<double>(((any_had ? 8ll : 4ll) * sms + nseq - 1) / nseq);
  Quant3VarArgs a;
  Quant3Args& q3 = a.q;
  q3.first[0] = 0;
  int max_h = 1;
  for (int i = 0; i < 3; ++i) {
    QuantArgs& t = q3.t[i];
    if (i >= n) {   // unused slots: no CTA columns
      t = q3.t[0];
      q3.had[i] = 0;
      q3.first[i + 1] = q3.first[i];
      continue;
    }
    long long chunks = static_cast<long long>(want * bytes[i] / total + 0.5);
    if (chunks < 1) chunks = 1;
    if (chunks > mean_len) chunks = mean_len;
    t.x = xs[i];
    t.out = static_cast<uint8_t*>(outs[i]);
    t.scale = scs[i];
    t.S = 0;
    t.H = Hs[i]; t.D = Ds[i];
    t.rows_per_cta = static_cast<int>(prepass_rows((mean_len + chunks - 1) / chunks, Hs[i], Ds[i]));
    set_div_magic(t, in_dtype);
    q3.had[i] = had[i];
    long long cols = 0;   // every sequence's chunks, in order
    for (int sq = 0; sq < nseq; ++sq) cols += (cu[sq + 1] - cu[sq] + t.rows_per_cta - 1) / t.rows_per_cta;
    if (q3.first[i] + cols > 0x7fffffffll) return ZYFA_ERR_BAD_SHAPE;
    q3.first[i + 1] = q3.first[i] + static_cast<int>(cols);
    max_h = std::max(max_h, Hs[i]);
  }
  a.n = nseq;
  for (int i = 0; i <= nseq; ++i) a.cu[i] = cu[i];
  const int n0 = nseq * Hs[0], n1 = n > 1 ? nseq * Hs[1] : 0, n2 = n > 2 ? nseq * Hs[2] : 0;
  const int nn = n0 + n1 + n2;
  float* s1 = n > 1 ? scs[1] : scs[0];
  float* s2 = n > 2 ? scs[2] : scs[0];
  // the zero step in plain stream order, the others as dependent launches
  quant3_zero_kernel<<<(nn + 255) / 256, 256, 0, st>>>(scs[0], s1, s2, n0, n1, n2);
  if (cudaGetLastError() != cudaSuccess) return ZYFA_ERR_CUDA;
  cudaError_t e = cudaSuccess;
  if (q3.first[3] > 0) {   // some sequence has rows
    const dim3 grid(static_cast<unsigned>(q3.first[3]), 1u), blk(kQuantThreads);
    const size_t shm = static_cast<size_t>(max_h) * 8;   // amax, or scale and its reciprocal, per head
    if (in_dtype == ZYFA_BF16) {
      e = launch_dependent(quant3v_amax_kernel<__nv_bfloat16>, grid, blk, shm, st, a);
      if (e == cudaSuccess) e = launch_dependent(quant3v_codes_kernel<__nv_bfloat16>, grid, blk, shm, st, a);
    } else {
      e = launch_dependent(quant3v_amax_kernel<float>, grid, blk, shm, st, a);
      if (e == cudaSuccess) e = launch_dependent(quant3v_codes_kernel<float>, grid, blk, shm, st, a);
    }
  }
  if (e == cudaSuccess)
    e = launch_dependent(quant3_finalize_kernel, dim3((nn + 255) / 256), dim3(256), 0, st, scs[0], s1, s2, n0, n1,
                         n2);
  if (e != cudaSuccess) return ZYFA_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? ZYFA_OK : ZYFA_ERR_CUDA;
}

extern "C" int zyfa_quantize_varlen(const void* x, int in_dtype, void* x_fp8, float* scale, const int* cu_seqlens,
                                    int nseq, int H, int D, int hadamard, void* stream) {
  const int badc = cu_validate(cu_seqlens, nseq, kMaxQuantSeqs);
  if (badc != ZYFA_OK) return badc;
  if (!scale || (cu_seqlens[nseq] > 0 && (!x || !x_fp8))) return ZYFA_ERR_NULL_PTR;
  if (H < 1 || H > 4096) return ZYFA_ERR_BAD_SHAPE;
  if (in_dtype != ZYFA_BF16 && in_dtype != ZYFA_FP32) return ZYFA_ERR_BAD_DTYPE;
  if (hadamard != 0 && hadamard != 1) return ZYFA_ERR_BAD_DTYPE;
  if (D < 8 || D > 1024 || D % 8 != 0 || (hadamard && D != 128 && D != 192)) return ZYFA_ERR_UNSUPPORTED_HEADDIM;
  if (!aligned(x, 16) || !aligned(x_fp8, 16) || !aligned(scale, 4)) return ZYFA_ERR_MISALIGNED;
  const void* xs[1] = {x};
  void* outs[1] = {x_fp8};
  float* scs[1] = {scale};
  const int Hs[1] = {H}, Ds[1] = {D}, had[1] = {hadamard};
  return quantize_varlen_n(1, xs, outs, scs, Hs, Ds, had, in_dtype, cu_seqlens, nseq, stream);
}

extern "C" int zyfa_quantize_qkv_varlen(const void* q, const void* k, const void* v, int in_dtype, void* q_fp8,
                                        void* k_fp8, void* v_fp8, float* q_scale, float* k_scale, float* v_scale,
                                        const int* cu_seqlens, int nseq, int Hq, int Hkv, int Dqk, int Dv,
                                        int hadamard_qk, void* stream) {
  const int badc = cu_validate(cu_seqlens, nseq, kMaxQuantSeqs);
  if (badc != ZYFA_OK) return badc;
  if (!q_scale || !k_scale || !v_scale) return ZYFA_ERR_NULL_PTR;
  if (cu_seqlens[nseq] > 0 && (!q || !k || !v || !q_fp8 || !k_fp8 || !v_fp8)) return ZYFA_ERR_NULL_PTR;
  if (Hq < 1 || Hkv < 1 || Hq > 4096 || Hkv > 4096) return ZYFA_ERR_BAD_SHAPE;
  if (in_dtype != ZYFA_BF16 && in_dtype != ZYFA_FP32) return ZYFA_ERR_BAD_DTYPE;
  if (hadamard_qk != 0 && hadamard_qk != 1) return ZYFA_ERR_BAD_DTYPE;
  for (int d : {Dqk, Dv})
    if (d < 8 || d > 1024 || d % 8 != 0) return ZYFA_ERR_UNSUPPORTED_HEADDIM;
  if (hadamard_qk && Dqk != 128 && Dqk != 192) return ZYFA_ERR_UNSUPPORTED_HEADDIM;
  for (const void* t : {q, k, v, static_cast<const void*>(q_fp8), static_cast<const void*>(k_fp8),
                        static_cast<const void*>(v_fp8)})
    if (!aligned(t, 16)) return ZYFA_ERR_MISALIGNED;
  if (!aligned(q_scale, 4) || !aligned(k_scale, 4) || !aligned(v_scale, 4)) return ZYFA_ERR_MISALIGNED;
  const void* xs[3] = {q, k, v};
  void* outs[3] = {q_fp8, k_fp8, v_fp8};
  float* scs[3] = {q_scale, k_scale, v_scale};
  const int Hs[3] = {Hq, Hkv, Hkv}, Ds[3] = {Dqk, Dqk, Dv}, had[3] = {hadamard_qk, hadamard_qk, 0};
  return quantize_varlen_n(3, xs, outs, scs, Hs, Ds, had, in_dtype, cu_seqlens, nseq, stream);
}

extern "C" int zyfa_attn_kv_tile(int dtype, int Dqk) {
  if (dtype != ZYFA_BF16 && dtype != ZYFA_FP8_E4M3) return ZYFA_ERR_BAD_DTYPE;
  if (Dqk != 128 && Dqk != 192) return ZYFA_ERR_UNSUPPORTED_HEADDIM;
  return (dtype == ZYFA_FP8_E4M3 && Dqk == 128) ? WideCfg::KT : 128;
}

extern "C" int zyfa_attn_schedule(int B, int S, const int* cu_seqlens, int Hq, int Hkv, int Dqk, int dtype,
                                  int grid, int cta, int* units, int cap) {
  if (Hq < 1 || Hkv < 1 || grid < 1 || cta < 0 || cta >= grid || cap < 0) return ZYFA_ERR_BAD_SHAPE;
  if (Hq % Hkv != 0) return ZYFA_ERR_BAD_GQA;
  if (Dqk != 128 && Dqk != 192) return ZYFA_ERR_UNSUPPORTED_HEADDIM;
  if (dtype != ZYFA_BF16 && dtype != ZYFA_FP8_E4M3) return ZYFA_ERR_BAD_DTYPE;
  if (cap > 0 && !units) return ZYFA_ERR_NULL_PTR;
  const int el = dtype == ZYFA_FP8_E4M3 ? 1 : 2;
  int n = 0, b, hkv, hq, qt, r0, len;
  auto put = [&]() {
    if (n < cap) { units[3 * n] = b; units[3 * n + 1] = hq; units[3 * n + 2] = qt; }
    ++n;
  };
  if (cu_seqlens) {
    const int badc = cu_validate(cu_seqlens, B, kMaxVarlenSeqs);
    if (badc != ZYFA_OK) return badc;
    if (varlen_units(cu_seqlens, B, Hq) > (1ll << 31) - 1) return ZYFA_ERR_BAD_SHAPE;
    VarlenSeqs t;
    fill_varlen_table(t, cu_seqlens, B, Dqk, el);
    VarlenIter it;
    it.init(grid, cta, &t, Hq, Hkv);
    while (it.next(b, hkv, hq, qt, r0, len)) put();
  } else {
    if (B < 1 || S < 1) return ZYFA_ERR_BAD_SHAPE;
    const long long tq = (static_cast<long long>(S) + 127) / 128;
    if (static_cast<long long>(B) * Hq * tq > (1ll << 31) - 1) return ZYFA_ERR_BAD_SHAPE;
    UnitIter it;
    it.init(grid, cta, static_cast<int>(tq), Hq, Hkv, B, group_slots_for(B, Hkv, S, Dqk, el));
    while (it.next(b, hkv, hq, qt)) put();
  }
  return n;
}

extern "C" int zyfa_device_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return ZYFA_ERR_CUDA;
  int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int)) != cudaSuccess) return ZYFA_ERR_CUDA;
  if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess) return ZYFA_ERR_CUDA;
  return v == kDevOk ? ZYFA_OK : ZYFA_ERR_DEVICE_TIMEOUT;
}

extern "C" int zyfa_device_check(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return ZYFA_ERR_CUDA;
  int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_check, sizeof(int)) != cudaSuccess) return ZYFA_ERR_CUDA;
  if (cudaMemcpyToSymbol(g_device_check, &zero, sizeof(int)) != cudaSuccess) return ZYFA_ERR_CUDA;
  return v;
}

extern "C" int zyfa_checked_build(void) { return kRangeChecks ? 1 : 0; }

extern "C" int zyfa_leanp_codes(const float* s, const float* m, const float* bmax, const float* A,
                                const unsigned char* masked, int n, unsigned char* code, int* j,
                                void* stream) {
  if (n < 0) return ZYFA_ERR_BAD_SHAPE;
  if (n == 0) return ZYFA_OK;
  if (!s || !m || !bmax || !A || !code) return ZYFA_ERR_NULL_PTR;
  const long long quads = (static_cast<long long>(n) + 3) / 4;
  const int blocks = static_cast<int>(std::min(1024ll, (quads + 255) / 256));
  leanp_codes_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(s, m, bmax, A, masked, n, code, j);
  return cudaGetLastError() == cudaSuccess ? ZYFA_OK : ZYFA_ERR_CUDA;
}

extern "C" int zyfa_selftest_wait_timeout(unsigned long long timeout_ns, void* stream) {
  if (timeout_ns > 1000000000ull) return ZYFA_ERR_BAD_SHAPE;
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(timeout_ns);
  return cudaGetLastError() == cudaSuccess ? ZYFA_OK : ZYFA_ERR_CUDA;
}

// C ABI of exattn: argument checks, TMA tensor maps and kernel launches.
// The operations themselves are documented in include/exattn.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <type_traits>
#include <algorithm>
#include <map>
#include <queue>
#include <tuple>
#include <vector>

#include "exattn.h"
#include "ptx.cuh"
#include "fwd.cuh"
#include "bwd.cuh"

namespace {

using exattn::BwdParams;
using exattn::FwdParams;

constexpr unsigned long long kDefaultTimeoutNs = 1000000000ull;  // 1 s per wait
constexpr int kMaxDevices = 64;
std::atomic<unsigned long long> g_timeout_ns{kDefaultTimeoutNs};  // see attn_set_wait_timeout_ns
std::atomic<unsigned int> g_debug_flags{0};                        // see attn_debug_inject_stall

// ------------------------------------------------------------------ checks
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// The kernels address rows of the [B*H, N padded to 128] views (the backward's
// accumulator, TMA row coordinates) with 32-bit ints, and the grids count
// 128-row tiles: both must stay below 2^31.  (A problem near the limit would
// need over 256 GB per tensor, more than the device holds.)
bool rows_fit(long long bh, int N) {
  const long long rows = (static_cast<long long>(N) + 127) / 128 * 128;
  return bh <= 0x7fffffffLL && rows * bh <= 0x7fffffffLL;
}

// 0 = proceed, 1 = empty problem (nothing to do), -1 = invalid
int check_sizes(int B, int H, int N, int d) {
  if (B < 0 || H < 0 || N < 0) return -1;
  if (d != 64 && d != 128) return -1;
  if (B == 0 || H == 0 || N == 0) return 1;
  return rows_fit(static_cast<long long>(B) * H, N) ? 0 : -1;
}

bool check_scale(float scale) { return std::isfinite(scale) && scale > 0.f; }

// Query rows per forward CTA: two 128-row sub-tiles, one at head_dim 256.
int fwd_rows(int d) { return d == 256 ? 128 : 256; }

// The forward also takes head_dim 256 (the backward does not).
int check_sizes_fwd(int B, int H, int N, int d) {
  if (d == 256) {
    if (B < 0 || H < 0 || N < 0) return -1;
    if (B == 0 || H == 0 || N == 0) return 1;
    return rows_fit(static_cast<long long>(B) * H, N) ? 0 : -1;
  }
  return check_sizes(B, H, N, d);
}

size_t padded_rows(int N) { return (static_cast<size_t>(N) + 127) / 128 * 128; }

struct Workspace {
  float* dq_acc;  // [BH, Np, d]
  float* dvec;    // [BH, Np]
  float* lse2;    // [BH, Np]
};

size_t workspace_bytes(int B, int H, int N, int d) {
  const size_t bh = static_cast<size_t>(B) * H;
  const size_t np = padded_rows(N);
  return bh * np * d * 4 + 2 * bh * np * 4;
}

Workspace carve(void* ws, int B, int H, int N, int d) {
  const size_t bh = static_cast<size_t>(B) * H;
  const size_t np = padded_rows(N);
  float* base = static_cast<float*>(ws);
  return Workspace{base, base + bh * np * d, base + bh * np * d + bh * np};
}

// ------------------------------------------------------------------ device
int check_device(int* dev_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ATTN_ERR_LAUNCH;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return ATTN_ERR_LAUNCH;
  if (major != 10 || minor != 0) return ATTN_ERR_UNSUPPORTED_DEVICE;
  if (dev < 0 || dev >= kMaxDevices) return ATTN_ERR_UNSUPPORTED_DEVICE;
  *dev_out = dev;
  return ATTN_OK;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                   CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(ptr);
  }();
  return fn;
}

template <typename T>
constexpr CUtensorMapDataType map_type() {
  if (sizeof(T) == 1) return CU_TENSOR_MAP_DATA_TYPE_UINT8;  // e4m3 bytes, copied as they are
  return std::is_same<T, __half>::value ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
}

// 3-D view {d, N, B*H} of a contiguous [B,H,N,d] tensor of T; box of 128
// bytes by 128 rows by 1 with 128-byte swizzle.  Rows past N of a head read
// as zeros.
template <typename T>
bool make_map_16(CUtensorMap* m, const void* base, int BH, int N, int d) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  constexpr cuuint64_t es = sizeof(T);
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * es, static_cast<cuuint64_t>(N) * d * es};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / es), 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, map_type<T>(), 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D view {d, rows} of the fp32 dQ accumulator [rows, d]; box {32, 32} with
// 128-byte swizzle, the target of the backward's TMA reduce-adds.
bool make_map_f32_dq(CUtensorMap* m, void* base, size_t rows, int d) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(d) * 4};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Opt-in to large dynamic shared memory, set before every launch: the
// attribute belongs to the loaded module, which a re-created context
// (cudaDeviceReset) loads afresh.  It is a host-side call.
template <typename K>
bool ensure_smem_attr(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess;
}

// The backward kernel rebalances registers between warpgroups (setmaxnreg);
// the split is only safe for a compiled register count in [kRegsMin, kRegsMax],
// so a build outside that range is refused before its first launch.
template <int D, typename T, bool kPersist>
bool bwd_regs_ok(int dev) {
  static std::atomic<int> checked[kMaxDevices];  // one table per kernel instantiation
  if (checked[dev].load(std::memory_order_acquire)) return true;
  cudaFuncAttributes a{};
  if (cudaFuncGetAttributes(&a, exattn::attn_bwd_kernel<D, T, kPersist>) != cudaSuccess) return false;
  if (a.numRegs < exattn::BwdCfg<D>::kRegsMin || a.numRegs > exattn::BwdCfg<D>::kRegsMax) return false;
  checked[dev].store(1, std::memory_order_release);
  return true;
}


int launch_status() { return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_LAUNCH; }

// Heads per scheduling group: the CTAs in flight then touch about
// kL2GroupBytes of per-head data, so that two groups fit in the 126 MB L2.
constexpr double kL2GroupBytes = 48.0 * 1024 * 1024;
int head_group(int BH, double per_head_bytes) {
  const double g = kL2GroupBytes / per_head_bytes;
  if (g >= BH) return BH;
  return g < 1.0 ? 1 : static_cast<int>(g);
}

// ------------------------------------------------------ typed implementations
// T is the 16-bit element type of the tensors: __nv_bfloat16 or __half.

// Launches the forward kernel for a filled-in parameter block (tensor maps
// and sizes set by the caller).
template <typename T>
int launch_fwd(FwdParams& p, int d, cudaStream_t s) {
  p.timeout_ns = g_timeout_ns.load(std::memory_order_relaxed);
  p.debug_flags = g_debug_flags.load(std::memory_order_relaxed);
  const dim3 grid(static_cast<unsigned>(p.nblocks) * static_cast<unsigned>(p.splits) * static_cast<unsigned>(p.BH));
  if constexpr (sizeof(T) == 1) {  // e4m3: head_dim 128 only
    if (d != 128) return ATTN_ERR_INVALID;
    constexpr int smem = exattn::FwdCfg<128, T>::kSmem;
    if (!ensure_smem_attr(exattn::attn_fwd_kernel<128, T>, smem)) return ATTN_ERR_LAUNCH;
    exattn::attn_fwd_kernel<128, T><<<grid, exattn::FwdCfg<128, T>::kThreads, smem, s>>>(p);
  } else if (d == 256) {
    constexpr int smem = exattn::FwdCfg<256, T>::kSmem;
    if (!ensure_smem_attr(exattn::attn_fwd_kernel<256, T>, smem)) return ATTN_ERR_LAUNCH;
    exattn::attn_fwd_kernel<256, T><<<grid, exattn::FwdCfg<256, T>::kThreads, smem, s>>>(p);
  } else if (d == 64) {
    constexpr int smem = exattn::FwdCfg<64, T>::kSmem;
    if (!ensure_smem_attr(exattn::attn_fwd_kernel<64, T>, smem)) return ATTN_ERR_LAUNCH;
    exattn::attn_fwd_kernel<64, T><<<grid, exattn::FwdCfg<64, T>::kThreads, smem, s>>>(p);
  } else {
    constexpr int smem = exattn::FwdCfg<128, T>::kSmem;
    if (!ensure_smem_attr(exattn::attn_fwd_kernel<128, T>, smem)) return ATTN_ERR_LAUNCH;
    exattn::attn_fwd_kernel<128, T><<<grid, exattn::FwdCfg<128, T>::kThreads, smem, s>>>(p);
  }
  return launch_status();
}

// The lean configuration (one sub-tile, two CTAs per SM) for a split-key
// forward with at most 128 query rows.
template <typename T>
int launch_fwd_lean(FwdParams& p, int d, cudaStream_t s) {
  p.timeout_ns = g_timeout_ns.load(std::memory_order_relaxed);
  p.debug_flags = g_debug_flags.load(std::memory_order_relaxed);
  const dim3 grid(static_cast<unsigned>(p.nblocks) * static_cast<unsigned>(p.splits) * static_cast<unsigned>(p.BH));
  if (d == 64) {
    using C = exattn::FwdCfg<64, T, true>;
    if (!ensure_smem_attr(exattn::attn_fwd_kernel<64, T, true>, C::kSmem)) return ATTN_ERR_LAUNCH;
    exattn::attn_fwd_kernel<64, T, true><<<grid, C::kThreads, C::kSmem, s>>>(p);
  } else {
    using C = exattn::FwdCfg<128, T, true>;
    if (!ensure_smem_attr(exattn::attn_fwd_kernel<128, T, true>, C::kSmem)) return ATTN_ERR_LAUNCH;
    exattn::attn_fwd_kernel<128, T, true><<<grid, C::kThreads, C::kSmem, s>>>(p);
  }
  return launch_status();
}

// Whether a split-key forward runs in the lean configuration.
bool use_lean(int Nq, int d, int elem_bytes) { return Nq <= 128 && d <= 128 && elem_bytes == 2; }

template <typename T>
int fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
             float scale, int causal, attn_stream_t stream) {
  const int sz = check_sizes_fwd(B, H, N, d);
  if (sz < 0 || !check_scale(scale)) return ATTN_ERR_INVALID;
  if (sz == 1) return ATTN_OK;
  if (!q || !k || !v || !o || !lse) return ATTN_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return ATTN_ERR_INVALID;
  int dev = 0;
  if (int st = check_device(&dev)) return st;

  FwdParams p;
  std::memset(&p, 0, sizeof(p));
  const int BH = B * H;
  if (!make_map_16<T>(&p.tm_q, q, BH, N, d) || !make_map_16<T>(&p.tm_k, k, BH, N, d) ||
      !make_map_16<T>(&p.tm_v, v, BH, N, d))
    return ATTN_ERR_LAUNCH;
  p.o = o;
  p.lse = lse;
  p.N = N;
  p.Nk = N;
  p.q_off = 0;
  p.BH = BH;
  p.nblocks = (N + fwd_rows(d) - 1) / fwd_rows(d);
  p.splits = 1;
  p.tps = (N + 127) / 128;
  p.head_group = head_group(BH, 2.0 * N * d * 2);  // K and V of one head
  p.causal = causal ? 1 : 0;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.o_mul = 1.0f;
  // Short rows: each CTA does few key tiles, so its fixed costs (Q load,
  // pipeline fill, epilogue) weigh; two lean CTAs per SM overlap them.
  // Measured on the sweep: +3% to +18% up to N = 1024, 3-7% slower from 2048.
  constexpr int kLeanMaxN = 1024;
  if (N <= kLeanMaxN && use_lean(1, d, sizeof(T))) {
    p.nblocks = (N + 127) / 128;
    return launch_fwd_lean<T>(p, d, reinterpret_cast<cudaStream_t>(stream));
  }
  return launch_fwd<T>(p, d, reinterpret_cast<cudaStream_t>(stream));
}

// e4m3 inputs: the per-tensor descale factors fold into the score scale (Q,
// K) and the output factor (V).
int fwd_fp8_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
                 float scale, int causal, float q_descale, float k_descale, float v_descale, attn_stream_t stream) {
  const int sz = check_sizes(B, H, N, d);
  if (sz < 0 || !check_scale(scale) || d != 128) return ATTN_ERR_INVALID;
  if (!check_scale(q_descale) || !check_scale(k_descale) || !check_scale(v_descale)) return ATTN_ERR_INVALID;
  const float eff = scale * q_descale * k_descale;
  if (!check_scale(eff)) return ATTN_ERR_INVALID;
  if (sz == 1) return ATTN_OK;
  if (!q || !k || !v || !o || !lse) return ATTN_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return ATTN_ERR_INVALID;
  int dev = 0;
  if (int st = check_device(&dev)) return st;
  FwdParams p;
  std::memset(&p, 0, sizeof(p));
  const int BH = B * H;
  if (!make_map_16<__nv_fp8_e4m3>(&p.tm_q, q, BH, N, d) || !make_map_16<__nv_fp8_e4m3>(&p.tm_k, k, BH, N, d) ||
      !make_map_16<__nv_fp8_e4m3>(&p.tm_v, v, BH, N, d))
    return ATTN_ERR_LAUNCH;
  p.o = o;
  p.lse = lse;
  p.N = N;
  p.Nk = N;
  p.q_off = 0;
  p.BH = BH;
  p.nblocks = (N + 255) / 256;
  p.splits = 1;
  p.tps = (N + 127) / 128;
  p.head_group = head_group(BH, 2.0 * N * d);  // K and V of one head
  p.causal = causal ? 1 : 0;
  p.scale = eff;
  p.scale_log2 = eff * 1.4426950408889634f;
  p.o_mul = v_descale;
  return launch_fwd<__nv_fp8_e4m3>(p, d, reinterpret_cast<cudaStream_t>(stream));
}

// ------------------------------------------------------ split-key forward
constexpr int kMaxSplits = 64;

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  return n;
}

// Key tiles that query block qb (256 rows) sees: all of them, or under the
// causal mask those up to the last visible key of its last row.
int block_tiles(int qb, int rows, int Nq, int Nk, int causal) {
  const int ntk = (Nk + 127) / 128;
  const int last = std::min(qb * rows + rows - 1, Nq - 1);
  return causal ? std::min(ntk, (last + (Nk - Nq)) / 128 + 1) : ntk;
}

// Number of key ranges per query block.  Enough CTAs for the machine come
// from the (batch, head, query block) grid when it holds four or more waves:
// then 1.  Otherwise each candidate S is simulated: the CTAs, in launch order
// (heaviest query block first), are handed to the SMs as they free up, a CTA
// costing its key tiles plus a fixed start-up cost, and S > 1 pays for the
// merge pass; the S with the shortest makespan wins.  The choice is made on
// whole tiles (Nq and Nk rounded up to the query block and the key tile), so
// that the calls of a decode loop, whose key count grows by one per step,
// share one plan per 128 keys; it depends only on those counts and the SM
// count and is cached (at most kMaxPlans entries; the cache starts over
// when full).
constexpr size_t kMaxPlans = 4096;
int choose_splits(int BH, int Nq, int Nk, int causal, int rows, int per_sm) {
  const int sms = sm_count() * per_sm;  // CTAs resident at once
  const int nblocks = (Nq + rows - 1) / rows;
  const int ntk = (Nk + 127) / 128;
  if (static_cast<long long>(BH) * nblocks >= 4LL * sms || ntk == 1) return 1;
  Nq = nblocks * rows;
  Nk = ntk * 128;
  static std::mutex mu;
  static std::map<std::tuple<int, int, int, int, int, int>, int> cache;
  const auto key = std::make_tuple(BH, nblocks, ntk, causal, sms, rows);  // sms counts resident CTAs
  {
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(key);
    if (it != cache.end()) return it->second;
  }
  constexpr double kStartup = 2.5;  // per CTA, in units of one key tile's time
  int best = 1;
  double best_cost = 0;
  for (int S = 1; S <= std::min(kMaxSplits, ntk); ++S) {
    const int tps = (ntk + S - 1) / S;
    const int se = (ntk + tps - 1) / tps;  // ranges actually distinct
    if (se != S) continue;
    if (static_cast<long long>(BH) * nblocks * S > 16LL * sms) break;
    std::priority_queue<double, std::vector<double>, std::greater<double>> free_at;
    for (int i = 0; i < sms; ++i) free_at.push(0.0);
    double makespan = 0;
    for (int r = 0; r < nblocks * S; ++r) {
      const int qb = nblocks - 1 - r / S, sp = r % S;
      const int cnt = std::max(0, std::min(block_tiles(qb, rows, Nq, Nk, causal) - sp * tps, tps));
      for (int h = 0; h < BH; ++h) {
        const double t = free_at.top() + cnt + kStartup;
        free_at.pop();
        free_at.push(t);
        makespan = std::max(makespan, t);
      }
    }
    // the merge reads and writes (d + 1) fp32 per row and range: a few tiles' time
    const double cost = makespan + (S > 1 ? 3.0 + 1e-6 * BH * static_cast<double>(Nq) * S : 0.0);
    if (S == 1 || cost < best_cost) {
      best = S;
      best_cost = cost;
    }
  }
  std::lock_guard<std::mutex> lock(mu);
  if (cache.size() >= kMaxPlans) cache.clear();
  cache[key] = best;
  return best;
}

// Resolves the split count (0 = automatic) and the key tiles per range.
void resolve_splits(int BH, int Nq, int Nk, int d, int elem_bytes, int causal, int requested, int* splits,
                    int* tps) {
  const int ntk = (Nk + 127) / 128;
  const bool lean = use_lean(Nq, d, elem_bytes);
  int S = requested > 0 ? std::min(requested, kMaxSplits)
                        : choose_splits(BH, Nq, Nk, causal, lean ? 128 : fwd_rows(d), lean ? 2 : 1);
  S = std::max(1, std::min(S, ntk));
  const int t = (ntk + S - 1) / S;
  *tps = t;
  *splits = (ntk + t - 1) / t;
}

size_t round_up256(size_t x) { return (x + 255) / 256 * 256; }

size_t kvsplit_ws_bytes(int BH, int Nq, int d, int S) {
  if (S <= 1) return 0;
  const size_t rows = static_cast<size_t>(BH) * S * Nq;
  return round_up256(rows * d * 4) + round_up256(rows * 4);
}

int check_kvsplit_sizes(int B, int H, int Nq, int Nk, int d, int causal, int splits) {
  if (Nk < 0 || splits < 0) return -1;
  const int sz = check_sizes_fwd(B, H, Nq, d);
  if (sz != 0) return sz;
  if (Nk == 0) return -1;             // a query with no keys has no softmax
  if (causal && Nq > Nk) return -1;  // the first rows would see no key
  const long long units = static_cast<long long>(B) * H * ((Nq + 127) / 128) * kMaxSplits;
  if (units > 0x7fffffffLL) return -1;
  return 0;
}

template <typename T>
int kvsplit_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Nq, int Nk,
                 int d, float scale, int causal, int splits, void* workspace, size_t workspace_bytes_given,
                 attn_stream_t stream) {
  const int sz = check_kvsplit_sizes(B, H, Nq, Nk, d, causal, splits);
  if (sz < 0 || !check_scale(scale)) return ATTN_ERR_INVALID;
  if (sz == 1) return ATTN_OK;
  if (!q || !k || !v || !o || !lse) return ATTN_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return ATTN_ERR_INVALID;
  int dev = 0;
  if (int st = check_device(&dev)) return st;
  const int BH = B * H;
  int S = 1, tps = 1;
  resolve_splits(BH, Nq, Nk, d, sizeof(T), causal ? 1 : 0, splits, &S, &tps);
  const size_t need = kvsplit_ws_bytes(BH, Nq, d, S);
  if (need > 0 && (!workspace || workspace_bytes_given < need || (reinterpret_cast<uintptr_t>(workspace) & 255u)))
    return ATTN_ERR_INVALID;

  FwdParams p;
  std::memset(&p, 0, sizeof(p));
  if (!make_map_16<T>(&p.tm_q, q, BH, Nq, d) || !make_map_16<T>(&p.tm_k, k, BH, Nk, d) ||
      !make_map_16<T>(&p.tm_v, v, BH, Nk, d))
    return ATTN_ERR_LAUNCH;
  p.o = o;
  p.lse = lse;
  p.N = Nq;
  p.Nk = Nk;
  p.q_off = Nk - Nq;
  const bool lean = use_lean(Nq, d, sizeof(T));
  p.BH = BH;
  p.nblocks = lean ? 1 : (Nq + fwd_rows(d) - 1) / fwd_rows(d);
  p.splits = S;
  p.tps = tps;
  if (S > 1) {
    const size_t rows = static_cast<size_t>(BH) * S * Nq;
    p.part_o = static_cast<float*>(workspace);
    p.part_lse = reinterpret_cast<float*>(static_cast<char*>(workspace) + round_up256(rows * d * 4));
  }
  p.head_group = head_group(BH, 2.0 * Nk * d * 2);
  p.causal = causal ? 1 : 0;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.o_mul = 1.0f;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (int st = lean ? launch_fwd_lean<T>(p, d, s) : launch_fwd<T>(p, d, s)) return st;
  if (S == 1) return ATTN_OK;
  const long long rows = static_cast<long long>(BH) * Nq;
  const unsigned blocks = static_cast<unsigned>((rows + 7) / 8);
  if (d == 64)
    exattn::attn_fwd_merge_kernel<64, T><<<blocks, 256, 0, s>>>(p.part_o, p.part_lse, o, lse, BH, Nq, S);
  else if (d == 128)
    exattn::attn_fwd_merge_kernel<128, T><<<blocks, 256, 0, s>>>(p.part_o, p.part_lse, o, lse, BH, Nq, S);
  else
    exattn::attn_fwd_merge_kernel<256, T><<<blocks, 256, 0, s>>>(p.part_o, p.part_lse, o, lse, BH, Nq, S);
  return launch_status();
}

template <typename T>
int preprocess_impl(const void* o, const void* dO, const float* lse, int B, int H, int N, int d,
                        void* workspace, size_t workspace_bytes_given, attn_stream_t stream) {
  const int sz = check_sizes(B, H, N, d);
  if (sz < 0) return ATTN_ERR_INVALID;
  if (sz == 1) return ATTN_OK;
  if (!o || !dO || !lse || !workspace) return ATTN_ERR_INVALID;
  if (!aligned16(o) || !aligned16(dO) || !aligned16(lse) || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return ATTN_ERR_INVALID;
  if (workspace_bytes_given < workspace_bytes(B, H, N, d)) return ATTN_ERR_INVALID;
  int dev = 0;
  if (int st = check_device(&dev)) return st;
  const Workspace ws = carve(workspace, B, H, N, d);
  const int BH = B * H;
  const int np = static_cast<int>(padded_rows(N));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  exattn::launch_bwd_preprocess<T>(o, dO, lse, ws.dvec, ws.lse2, ws.dq_acc, BH, N, np, d, s);
  return launch_status();
}

// Key tiles per head up to which the main backward runs persistent CTAs
// (measured against one CTA per key tile): at head_dim 128, 8 (N <= 1024;
// +10 to +14%) and 16 under the causal mask (+3%; -1% without it); at
// head_dim 64, 32 (+1 to +4%) and 64 under the causal mask (+2%; -0.5%
// without it).
bool bwd_persistent(int ntiles, int d, int causal) {
  if (d == 64) return ntiles <= (causal ? 64 : 32);
  return ntiles <= (causal ? 16 : 8);
}

template <int D, typename T, bool kPersist>
int launch_bwd(const BwdParams& p, dim3 grid, int dev, cudaStream_t s) {
  constexpr int smem = exattn::BwdCfg<D>::kSmem;
  if (!bwd_regs_ok<D, T, kPersist>(dev)) return ATTN_ERR_LAUNCH;
  if (!ensure_smem_attr(exattn::attn_bwd_kernel<D, T, kPersist>, smem)) return ATTN_ERR_LAUNCH;
  exattn::attn_bwd_kernel<D, T, kPersist><<<grid, exattn::BwdCfg<D>::kThreads, smem, s>>>(p);
  return launch_status();
}

template <typename T>
int dkdv_impl(const void* q, const void* k, const void* v, const void* dO, void* dk, void* dv, int B, int H,
                  int N, int d, float scale, int causal, void* workspace, size_t workspace_bytes_given,
                  attn_stream_t stream) {
  const int sz = check_sizes(B, H, N, d);
  if (sz < 0 || !check_scale(scale)) return ATTN_ERR_INVALID;
  if (sz == 1) return ATTN_OK;
  if (!q || !k || !v || !dO || !dk || !dv || !workspace) return ATTN_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dO) || !aligned16(dk) || !aligned16(dv) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return ATTN_ERR_INVALID;
  if (workspace_bytes_given < workspace_bytes(B, H, N, d)) return ATTN_ERR_INVALID;
  int dev = 0;
  if (int st = check_device(&dev)) return st;
  const Workspace ws = carve(workspace, B, H, N, d);
  BwdParams p;
  std::memset(&p, 0, sizeof(p));
  const int BH = B * H;
  if (!make_map_16<T>(&p.tm_q, q, BH, N, d) || !make_map_16<T>(&p.tm_k, k, BH, N, d) ||
      !make_map_16<T>(&p.tm_v, v, BH, N, d) || !make_map_16<T>(&p.tm_do, dO, BH, N, d) ||
      !make_map_f32_dq(&p.tm_dq, ws.dq_acc, static_cast<size_t>(BH) * padded_rows(N), d))
    return ATTN_ERR_LAUNCH;
  p.dk = dk;
  p.dv = dv;
  p.dq_acc = ws.dq_acc;
  p.dvec = ws.dvec;
  p.lse2 = ws.lse2;
  p.N = N;
  p.Np = static_cast<int>(padded_rows(N));
  p.BH = BH;
  p.ntiles = (N + 127) / 128;
  p.head_group = head_group(BH, 2.0 * N * d * 2 + 4.0 * N * d);  // Q, dO (bf16) and the dQ rows (fp32)
  p.causal = causal ? 1 : 0;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.timeout_ns = g_timeout_ns.load(std::memory_order_relaxed);
  p.debug_flags = g_debug_flags.load(std::memory_order_relaxed);
  // Short rows (see bwd_persistent), where a CTA's start-up and
  // epilogue are a large share of its few steps: persistent
  // CTAs, one per SM (the kernel's TMEM and shared memory allow no second),
  // each walking the work units (a key tile, or under the causal mask a pair
  // of key tiles, of one head) with a stride of the grid.  Longer rows: one
  // CTA per key tile, handed out by the hardware as SMs free up (measured
  // faster there).
  const bool persist = bwd_persistent(p.ntiles, d, causal);
  p.paired = (persist && causal) ? 1 : 0;
  const long long units = static_cast<long long>(p.paired ? (p.ntiles + 1) / 2 : p.ntiles) * BH;
  const dim3 grid(static_cast<unsigned>(persist ? std::min<long long>(units, sm_count()) : units));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (d == 64)
    return persist ? launch_bwd<64, T, true>(p, grid, dev, s) : launch_bwd<64, T, false>(p, grid, dev, s);
  return persist ? launch_bwd<128, T, true>(p, grid, dev, s) : launch_bwd<128, T, false>(p, grid, dev, s);
}

template <typename T>
int dq_convert_impl(void* dq, int B, int H, int N, int d, float scale, const void* workspace,
                        size_t workspace_bytes_given, attn_stream_t stream) {
  const int sz = check_sizes(B, H, N, d);
  if (sz < 0 || !check_scale(scale)) return ATTN_ERR_INVALID;
  if (sz == 1) return ATTN_OK;
  if (!dq || !workspace) return ATTN_ERR_INVALID;
  if (!aligned16(dq) || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return ATTN_ERR_INVALID;
  if (workspace_bytes_given < workspace_bytes(B, H, N, d)) return ATTN_ERR_INVALID;
  int dev = 0;
  if (int st = check_device(&dev)) return st;
  const Workspace ws = carve(const_cast<void*>(workspace), B, H, N, d);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  exattn::launch_bwd_dq_convert<T>(ws.dq_acc, dq, B * H, N, static_cast<int>(padded_rows(N)), d, scale, s);
  return launch_status();
}

template <typename T>
int bwd_impl(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
             void* dq, void* dk, void* dv, int B, int H, int N, int d, float scale, int causal, void* workspace,
             size_t workspace_bytes_given, attn_stream_t stream) {
  const int sz = check_sizes(B, H, N, d);
  if (sz < 0 || !check_scale(scale)) return ATTN_ERR_INVALID;
  if (sz == 1) return ATTN_OK;
  if (!dq) return ATTN_ERR_INVALID;
  int st = preprocess_impl<T>(o, dO, lse, B, H, N, d, workspace, workspace_bytes_given, stream);
  if (st) return st;
  st = dkdv_impl<T>(q, k, v, dO, dk, dv, B, H, N, d, scale, causal, workspace, workspace_bytes_given, stream);
  if (st) return st;
  return dq_convert_impl<T>(dq, B, H, N, d, scale, workspace, workspace_bytes_given, stream);
}

}  // namespace

extern "C" {

// ------------------------------------------------------------- bf16 entry points
int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
             float scale, int causal, attn_stream_t stream) {
  return fwd_impl<__nv_bfloat16>(q, k, v, o, lse, B, H, N, d, scale, causal, stream);
}

size_t attn_bwd_workspace_bytes(int B, int H, int N, int d) {
  if (check_sizes(B, H, N, d) != 0) return 0;
  return workspace_bytes(B, H, N, d);
}

int attn_bwd_preprocess(const void* o, const void* dO, const float* lse, int B, int H, int N, int d,
                        void* workspace, size_t workspace_bytes_given, attn_stream_t stream) {
  return preprocess_impl<__nv_bfloat16>(o, dO, lse, B, H, N, d, workspace, workspace_bytes_given, stream);
}

int attn_bwd_dkdv(const void* q, const void* k, const void* v, const void* dO, void* dk, void* dv, int B, int H,
                  int N, int d, float scale, int causal, void* workspace, size_t workspace_bytes_given,
                  attn_stream_t stream) {
  return dkdv_impl<__nv_bfloat16>(q, k, v, dO, dk, dv, B, H, N, d, scale, causal, workspace,
                                  workspace_bytes_given, stream);
}

int attn_bwd_dq_convert(void* dq, int B, int H, int N, int d, float scale, const void* workspace,
                        size_t workspace_bytes_given, attn_stream_t stream) {
  return dq_convert_impl<__nv_bfloat16>(dq, B, H, N, d, scale, workspace, workspace_bytes_given, stream);
}

int attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
             void* dq, void* dk, void* dv, int B, int H, int N, int d, float scale, int causal, void* workspace,
             size_t workspace_bytes_given, attn_stream_t stream) {
  return bwd_impl<__nv_bfloat16>(q, k, v, o, lse, dO, dq, dk, dv, B, H, N, d, scale, causal, workspace,
                                 workspace_bytes_given, stream);
}

// ------------------------------------------------------------- split-key forward
size_t attn_fwd_kvsplit_workspace_bytes(int B, int H, int Nq, int Nk, int d, int causal, int splits) {
  if (check_kvsplit_sizes(B, H, Nq, Nk, d, causal, splits) != 0) return 0;
  int S = 1, tps = 1;
  resolve_splits(B * H, Nq, Nk, d, 2, causal ? 1 : 0, splits, &S, &tps);
  return kvsplit_ws_bytes(B * H, Nq, d, S);
}

int attn_fwd_kvsplit_count(int B, int H, int Nq, int Nk, int d, int causal, int splits) {
  if (check_kvsplit_sizes(B, H, Nq, Nk, d, causal, splits) != 0) return 0;
  int S = 1, tps = 1;
  resolve_splits(B * H, Nq, Nk, d, 2, causal ? 1 : 0, splits, &S, &tps);
  return S;
}

int attn_fwd_kvsplit(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Nq,
                     int Nk, int d, float scale, int causal, int splits, void* workspace,
                     size_t workspace_bytes_given, attn_stream_t stream) {
  return kvsplit_impl<__nv_bfloat16>(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal, splits, workspace,
                                     workspace_bytes_given, stream);
}

int attn_fwd_kvsplit_fp16(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Nq,
                          int Nk, int d, float scale, int causal, int splits, void* workspace,
                          size_t workspace_bytes_given, attn_stream_t stream) {
  return kvsplit_impl<__half>(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal, splits, workspace,
                              workspace_bytes_given, stream);
}

// ------------------------------------------------------------- e4m3 forward
int attn_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
                 float scale, int causal, float q_descale, float k_descale, float v_descale, attn_stream_t stream) {
  return fwd_fp8_impl(q, k, v, o, lse, B, H, N, d, scale, causal, q_descale, k_descale, v_descale, stream);
}

// ------------------------------------------------------------- fp16 entry points
int attn_fwd_fp16(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
                  float scale, int causal, attn_stream_t stream) {
  return fwd_impl<__half>(q, k, v, o, lse, B, H, N, d, scale, causal, stream);
}

int attn_bwd_fp16(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                  void* dq, void* dk, void* dv, int B, int H, int N, int d, float scale, int causal,
                  void* workspace, size_t workspace_bytes_given, attn_stream_t stream) {
  return bwd_impl<__half>(q, k, v, o, lse, dO, dq, dk, dv, B, H, N, d, scale, causal, workspace,
                          workspace_bytes_given, stream);
}

void attn_set_wait_timeout_ns(unsigned long long ns) {
  g_timeout_ns.store(ns == 0 ? kDefaultTimeoutNs : ns, std::memory_order_relaxed);
}

void attn_debug_inject_stall(int on) {
  g_debug_flags.store(on ? exattn::kDebugSkipFirstKV : 0u, std::memory_order_relaxed);
}

int attn_get_device_status(attn_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return ATTN_ERR_LAUNCH;
  unsigned int word = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&word, exattn::g_status_word, sizeof(word)) != cudaSuccess) return ATTN_ERR_LAUNCH;
  if (word == 0) return ATTN_OK;
  if (cudaMemcpyToSymbol(exattn::g_status_word, &zero, sizeof(zero)) != cudaSuccess ||
      cudaMemcpyToSymbol(exattn::g_status_site, &zero, sizeof(zero)) != cudaSuccess)
    return ATTN_ERR_LAUNCH;
  return (word & exattn::kDevStatusTimeout) ? ATTN_ERR_TIMEOUT : ATTN_ERR_LAUNCH;
}

const char* attn_status_string(int status) {
  switch (status) {
    case ATTN_OK: return "ATTN_OK";
    case ATTN_ERR_INVALID: return "ATTN_ERR_INVALID";
    case ATTN_ERR_UNSUPPORTED_DEVICE: return "ATTN_ERR_UNSUPPORTED_DEVICE";
    case ATTN_ERR_LAUNCH: return "ATTN_ERR_LAUNCH";
    case ATTN_ERR_TIMEOUT: return "ATTN_ERR_TIMEOUT";
    default: return "ATTN_ERR_UNKNOWN";
  }
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Backward with library-owned scratch: attn_bwd_noalloc().
//
// For callers that must not allocate device memory themselves: code that
// runs with a fixed device-memory budget settled at start-up, plugins whose
// host application owns the device allocator, and code paths where a
// cudaMalloc/cudaFree (which may synchronise the whole device) is not
// allowed.  The backward's scratch (fp32 dQ accumulator plus two fp32 row
// vectors) lives in one file-scope __device__ array of
// EXATTN_NOALLOC_SCRATCH_BYTES, which every GPU that loads this library holds
// until the process exits.  In host code the array's name is only a host-side
// stand-in, so its device address is fetched with cudaGetSymbolAddress, on
// every call with the caller's device current, and passed to the kernels.
// ---------------------------------------------------------------------------
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[EXATTN_NOALLOC_SCRATCH_BYTES];

// The array's device address in the current device's context.  It is looked
// up on every call rather than cached: after cudaDeviceReset (or any other
// re-creation of the primary context) the module is loaded again and the
// array may sit at a different address.  The lookup is a host-side table
// read, no device work.
int noalloc_scratch_address(void** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return ATTN_ERR_LAUNCH;
  *out = p;
  return ATTN_OK;
}

}  // namespace

extern "C" int attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                                const void* dO, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                                float scale, int causal, attn_stream_t stream) {
  const int sz = check_sizes(B, H, N, d);
  if (sz < 0 || !check_scale(scale)) return ATTN_ERR_INVALID;
  if (sz == 1) return ATTN_OK;
  if (workspace_bytes(B, H, N, d) > static_cast<size_t>(EXATTN_NOALLOC_SCRATCH_BYTES)) return ATTN_ERR_INVALID;
  int dev = 0;
  if (int st = check_device(&dev)) return st;
  void* scratch = nullptr;
  if (int st = noalloc_scratch_address(&scratch)) return st;
  return attn_bwd(q, k, v, o, lse, dO, dq, dk, dv, B, H, N, d, scale, causal, scratch,
                  static_cast<size_t>(EXATTN_NOALLOC_SCRATCH_BYTES), stream);
}

// ---------------------------------------------------------------------------
// Forward + backward over host-resident tensors: attn_fwd_bwd_host().
//
// The (batch, head) pairs are split into chunks; chunk c uses buffer set
// c % kHostStages of the caller's device buffer.  Per chunk, on three streams:
//   copy-in stream:  [wait: set free] H2D q, k, v, dO      -> in_done[set]
//   caller's stream: [wait: in_done] fwd -> fwd_done[set], bwd -> bwd_done[set]
//   copy-out stream: [wait: fwd_done] D2H o, lse; [wait: bwd_done] D2H dq, dk,
//                    dv -> free[set]
// Events are recorded and waited on in host order, so each wait sees the
// record of the same chunk.  Entry and exit are tied to the caller's stream.
// ---------------------------------------------------------------------------
namespace {

// Three buffer sets: chunk c+1 is copied in while chunk c computes and chunk
// c-1 is copied out, without waiting for the copy-out of c-1 (as two sets
// would), so the two PCIe directions run independently.
constexpr int kHostStages = 3;

struct HostPipe {
  bool ready = false;
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t start = nullptr, end = nullptr;
  cudaEvent_t in_done[kHostStages] = {}, fwd_done[kHostStages] = {}, bwd_done[kHostStages] = {},
              free_[kHostStages] = {};
};

std::mutex g_pipe_mu;  // guards g_pipe and serialises the enqueue sequences that use it
HostPipe g_pipe[kMaxDevices];

int pipe_for(int dev, HostPipe** out) {
  HostPipe& hp = g_pipe[dev];
  if (!hp.ready) {
    const unsigned ef = cudaEventDisableTiming;
    bool ok = cudaStreamCreateWithFlags(&hp.in, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&hp.out, cudaStreamNonBlocking) == cudaSuccess &&
              cudaEventCreateWithFlags(&hp.start, ef) == cudaSuccess &&
              cudaEventCreateWithFlags(&hp.end, ef) == cudaSuccess;
    for (int s = 0; ok && s < kHostStages; ++s)
      ok = cudaEventCreateWithFlags(&hp.in_done[s], ef) == cudaSuccess &&
           cudaEventCreateWithFlags(&hp.fwd_done[s], ef) == cudaSuccess &&
           cudaEventCreateWithFlags(&hp.bwd_done[s], ef) == cudaSuccess &&
           cudaEventCreateWithFlags(&hp.free_[s], ef) == cudaSuccess;
    if (!ok) return ATTN_ERR_LAUNCH;
    hp.ready = true;
  }
  *out = &hp;
  return ATTN_OK;
}

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

int chunk_pairs(int BH, int heads_per_chunk) {
  if (heads_per_chunk > 0) return heads_per_chunk < BH ? heads_per_chunk : BH;
  return (BH + 7) / 8;
}

// one buffer set: q, k, v, dO, o, dq, dk, dv, lse, backward workspace
size_t stage_bytes(int G, int N, int d) {
  const size_t t = round256(static_cast<size_t>(G) * N * d * 2);
  return 8 * t + round256(static_cast<size_t>(G) * N * 4) + round256(workspace_bytes(1, G, N, d));
}

struct Stage {
  char *q, *k, *v, *dO, *o, *dq, *dk, *dv;
  float* lse;
  void* ws;
  size_t ws_bytes;
};

Stage carve_stage(char* base, int G, int N, int d) {
  const size_t t = round256(static_cast<size_t>(G) * N * d * 2);
  Stage s;
  char** slots[8] = {&s.q, &s.k, &s.v, &s.dO, &s.o, &s.dq, &s.dk, &s.dv};
  for (int i = 0; i < 8; ++i) *slots[i] = base + i * t;
  s.lse = reinterpret_cast<float*>(base + 8 * t);
  s.ws = base + 8 * t + round256(static_cast<size_t>(G) * N * 4);
  s.ws_bytes = workspace_bytes(1, G, N, d);
  return s;
}

}  // namespace

namespace {
int enqueue_host_chunks(HostPipe* hp, const void* q, const void* k, const void* v, const void* dO, void* o,
                        float* lse, void* dq, void* dk, void* dv, int N, int d, float scale, int causal,
                        char* dev_buf, int G, int nchunks, int BH, size_t sbytes, size_t row, attn_stream_t stream);
}  // namespace

extern "C" size_t attn_fwd_bwd_host_buffer_bytes(int B, int H, int N, int d, int heads_per_chunk) {
  if (check_sizes(B, H, N, d) != 0 || heads_per_chunk < 0) return 0;
  const int BH = B * H;
  const int G = chunk_pairs(BH, heads_per_chunk);
  const int stages = (BH + G - 1) / G < kHostStages ? (BH + G - 1) / G : kHostStages;
  return static_cast<size_t>(stages) * stage_bytes(G, N, d);
}

extern "C" int attn_fwd_bwd_host(const void* q, const void* k, const void* v, const void* dO, void* o, float* lse,
                                 void* dq, void* dk, void* dv, int B, int H, int N, int d, float scale, int causal,
                                 void* dev_buf, size_t dev_buf_bytes, int heads_per_chunk, attn_stream_t stream) {
  const int sz = check_sizes(B, H, N, d);
  if (sz < 0 || !check_scale(scale) || heads_per_chunk < 0) return ATTN_ERR_INVALID;
  if (sz == 1) return ATTN_OK;
  if (!q || !k || !v || !dO || !o || !lse || !dq || !dk || !dv || !dev_buf) return ATTN_ERR_INVALID;
  if ((reinterpret_cast<uintptr_t>(dev_buf) & 255u) != 0) return ATTN_ERR_INVALID;
  if (dev_buf_bytes < attn_fwd_bwd_host_buffer_bytes(B, H, N, d, heads_per_chunk)) return ATTN_ERR_INVALID;
  int dev = 0;
  if (int st = check_device(&dev)) return st;

  const int BH = B * H;
  const int G = chunk_pairs(BH, heads_per_chunk);
  const int nchunks = (BH + G - 1) / G;
  const size_t sbytes = stage_bytes(G, N, d);
  const size_t row = static_cast<size_t>(N) * d * 2;  // bytes of one (batch, head) of a bf16 tensor
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);

  std::lock_guard<std::mutex> lock(g_pipe_mu);
  HostPipe* hp = nullptr;
  if (int st = pipe_for(dev, &hp)) return st;
  auto ok = [](cudaError_t e) { return e == cudaSuccess; };
  if (!ok(cudaEventRecord(hp->start, cs)) || !ok(cudaStreamWaitEvent(hp->in, hp->start, 0)) ||
      !ok(cudaStreamWaitEvent(hp->out, hp->start, 0)))
    return ATTN_ERR_LAUNCH;
  const int st = enqueue_host_chunks(hp, q, k, v, dO, o, lse, dq, dk, dv, N, d, scale, causal,
                                     static_cast<char*>(dev_buf), G, nchunks, BH, sbytes, row, stream);
  // The caller's stream waits for everything enqueued above, also after a
  // failure part-way, so that no copy still runs once the caller may free or
  // reuse its buffers.
  const bool tied = ok(cudaEventRecord(hp->end, hp->in)) && ok(cudaStreamWaitEvent(cs, hp->end, 0)) &&
                    ok(cudaEventRecord(hp->end, hp->out)) && ok(cudaStreamWaitEvent(cs, hp->end, 0));
  if (st != ATTN_OK) return st;
  return tied ? ATTN_OK : ATTN_ERR_LAUNCH;
}

namespace {
int enqueue_host_chunks(HostPipe* hp, const void* q, const void* k, const void* v, const void* dO, void* o,
                        float* lse, void* dq, void* dk, void* dv, int N, int d, float scale, int causal,
                        char* dev_buf, int G, int nchunks, int BH, size_t sbytes, size_t row, attn_stream_t stream) {
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  auto ok = [](cudaError_t e) { return e == cudaSuccess; };
  for (int c = 0; c < nchunks; ++c) {
    const int s = c % kHostStages;
    const int h0 = c * G;
    const int g = (BH - h0) < G ? (BH - h0) : G;
    const size_t off = static_cast<size_t>(h0) * row, bytes = static_cast<size_t>(g) * row;
    const size_t loff = static_cast<size_t>(h0) * N, lbytes = static_cast<size_t>(g) * N * 4;
    const Stage st = carve_stage(dev_buf + s * sbytes, G, N, d);
    // copy in, once chunk c - kHostStages has left this buffer set
    if (c >= kHostStages && !ok(cudaStreamWaitEvent(hp->in, hp->free_[s], 0))) return ATTN_ERR_LAUNCH;
    const void* src[4] = {q, k, v, dO};
    char* dst[4] = {st.q, st.k, st.v, st.dO};
    for (int i = 0; i < 4; ++i)
      if (!ok(cudaMemcpyAsync(dst[i], static_cast<const char*>(src[i]) + off, bytes, cudaMemcpyHostToDevice,
                              hp->in)))
        return ATTN_ERR_LAUNCH;
    if (!ok(cudaEventRecord(hp->in_done[s], hp->in))) return ATTN_ERR_LAUNCH;
    // kernels on the caller's stream
    if (!ok(cudaStreamWaitEvent(cs, hp->in_done[s], 0))) return ATTN_ERR_LAUNCH;
    if (int e = attn_fwd(st.q, st.k, st.v, st.o, st.lse, 1, g, N, d, scale, causal, stream)) return e;
    if (!ok(cudaEventRecord(hp->fwd_done[s], cs))) return ATTN_ERR_LAUNCH;
    if (int e = attn_bwd(st.q, st.k, st.v, st.o, st.lse, st.dO, st.dq, st.dk, st.dv, 1, g, N, d, scale, causal,
                         st.ws, st.ws_bytes, stream))
      return e;
    if (!ok(cudaEventRecord(hp->bwd_done[s], cs))) return ATTN_ERR_LAUNCH;
    // copy out: O and LSE as soon as the forward is done, the gradients after the backward
    if (!ok(cudaStreamWaitEvent(hp->out, hp->fwd_done[s], 0)) ||
        !ok(cudaMemcpyAsync(static_cast<char*>(o) + off, st.o, bytes, cudaMemcpyDeviceToHost, hp->out)) ||
        !ok(cudaMemcpyAsync(lse + loff, st.lse, lbytes, cudaMemcpyDeviceToHost, hp->out)) ||
        !ok(cudaStreamWaitEvent(hp->out, hp->bwd_done[s], 0)))
      return ATTN_ERR_LAUNCH;
    void* hdst[3] = {dq, dk, dv};
    const char* dsrc[3] = {st.dq, st.dk, st.dv};
    for (int i = 0; i < 3; ++i)
      if (!ok(cudaMemcpyAsync(static_cast<char*>(hdst[i]) + off, dsrc[i], bytes, cudaMemcpyDeviceToHost, hp->out)))
        return ATTN_ERR_LAUNCH;
    if (!ok(cudaEventRecord(hp->free_[s], hp->out))) return ATTN_ERR_LAUNCH;
  }
  return ATTN_OK;
}
}  // namespace


// Forward kernel: O = softmax(scale Q K^T) V and LSE, tile by tile with an
// online softmax ("11.11 Flash Attention", sections "Flash Attention: The Key
// Insight" and "The Tiling Algorithm"; loop order of section "Flash
// Attention 2": Q blocks outside, K/V blocks inside, parallel over batch x
// heads x Q blocks).
//
// One CTA owns a 256-row block of queries of one (batch, head), split into two
// 128-row sub-tiles that ping-pong on the tensor core (while the softmax of
// one sub-tile runs, the MMAs of the other do).  At head_dim 256 a CTA owns one
// 128-row sub-tile (warps 0..3 softmax, 4 producer, 5 MMA): its O accumulator
// takes 256 TMEM columns.  Roles (320 threads):
//   warps 0..3    softmax of sub-tile 0 (one thread per query row)
//   warps 4..7    softmax of sub-tile 1
//   warp 8        TMA producer: Q (once), then K_j and V_j into a smem ring
//   warp 9        TMEM allocator; lane 0 issues every tcgen05.mma
// Tensor memory (512 columns x 128 lanes of 32 bit), per sub-tile k:
//   columns [256k, 256k+128)      S_k = Q_k K_j^T (fp32); P_k (16-bit pairs) is
//                                 written back over its first 64 columns
//   columns [256k+128, +d)        O_k accumulator (fp32; d = 256: columns 128..383)
// The softmax keeps, per row, a reference maximum and the running sum l;
// the division by l happens once at the end (section "Flash Attention 2":
// fewer non-matmul operations).  The reference maximum only moves when a
// tile's maximum exceeds it by more than 2^8 in probability units, so O is
// rescaled in TMEM rarely; this is exact, because O and l always share the
// same reference.
#pragma once
#include "ptx.cuh"

namespace exattn {

struct FwdParams {
  CUtensorMap tm_q;  // 3-D {d, N, B*H}, box {64, 128, 1}, 128-byte swizzle
  CUtensorMap tm_k;  // 3-D {d, Nk, B*H}, same boxes
  CUtensorMap tm_v;
  void* o;  // [B*H, N, d] of the element type T
  float* lse;
  int N;      // query rows per head
  int Nk;     // key rows per head (N for the square problem)
  int q_off;  // Nk - N: the causal mask lets query row r see keys <= r + q_off
  int BH;
  int nblocks;  // ceil(N / 256)
  int splits;   // key ranges per query block (1: the whole row, written as final output)
  int tps;      // key tiles per range
  float* part_o;    // splits > 1: [B*H, splits, N, d] fp32 partial O (normalised by its own l)
  float* part_lse;  // splits > 1: [B*H, splits, N] fp32 partial LSE (-inf where the range saw no key)
  int head_group;  // heads whose CTAs are scheduled together (L2 reuse of K/V)
  int causal;
  float scale;       // softmax scale (times the Q and K descale factors for e4m3 inputs)
  float scale_log2;  // scale * log2(e)
  float o_mul;       // factor applied to O on output (the V descale factor for e4m3 inputs, else 1)
  unsigned long long timeout_ns;
  unsigned int debug_flags;
};

// Exponential pairs (out of every 8) evaluated by ex2_fma on the FMA pipe;
// the special-function unit alone cannot keep pace with the tensor core at
// d = 128 (one exp per score against 4*d flops of MMA).
constexpr int kEmuPairs = 3;

// T: the input element type (16-bit, or e4m3).  A tile row holds D
// elements; tiles are stored as 128-byte swizzled chunks of 128 rows.
// kLean: a CTA of one 128-row sub-tile with a 2-slot K/V ring and 256 TMEM
// columns, small enough that two CTAs share an SM.  For few query rows
// (decode), where a second sub-tile would have no rows to work on, two such
// CTAs keep the tensor core and the softmax of an SM overlapping.
template <int D, typename T, bool kLean = false>
struct FwdCfg {
  // 128-row query sub-tiles per CTA: two, except at head_dim 256, where one
  // sub-tile's S (128 columns) and O (256) already take 384 of the 512 TMEM
  // columns, and in the lean configuration.
  static constexpr int kSub = (D == 256 || kLean) ? 1 : 2;
  static_assert(!kLean || (D <= 128 && sizeof(T) == 2), "lean CTAs: 16-bit inputs, head_dim <= 128");
  static constexpr uint32_t kTmemCols = kLean ? 256u : 512u;
  static constexpr int kCtasPerSm = kLean ? 2 : 1;
  static constexpr int kRows = 128 * kSub;                     // query rows per CTA
  static constexpr int kThreads = 128 * kSub + 64;             // softmax warps, producer warp, MMA warp
  static constexpr uint32_t kElem = sizeof(T);
  static constexpr uint32_t kTile = 128u * D * kElem;          // one 128-row tile
  // K/V ring slots within the 227 KB of shared memory
  static constexpr int kSlots = kLean ? 2 : (kTile == 65536u) ? 2 : (kTile == 32768u) ? 4 : 8;
  static constexpr int kChunks = D * kElem / 128;              // 128-byte swizzle chunks per row
  static constexpr int kChunkElems = 128 / kElem;              // elements per chunk
  static constexpr int kKStep = 32 / kElem;                    // K of one MMA (32 bytes of a row)
  static constexpr int kSSteps = D / kKStep;                   // MMAs of one S product
  static constexpr int kPVSteps = 128 / kKStep;                // MMAs of one P V product (128 keys)
  static constexpr int kPCols = 128 * kElem / 4;               // TMEM columns of P (128 keys)
  static constexpr uint32_t kBarOff = (kSub + kSlots) * kTile;
  static constexpr uint32_t kSmem = kBarOff + 256;
};

// T: the element type of Q, K and V (__nv_bfloat16, __half, or __nv_fp8_e4m3);
// O has type Elem<T>::Out.
template <int D, typename T, bool kLean = false>
__global__ void __launch_bounds__(FwdCfg<D, T, kLean>::kThreads, FwdCfg<D, T, kLean>::kCtasPerSm)
    attn_fwd_kernel(const __grid_constant__ FwdParams p) {
  using C = FwdCfg<D, T, kLean>;
  using E = Elem<T>;
  using TO = typename E::Out;
  constexpr int kProducerWarp = 4 * C::kSub;
  constexpr int kMmaWarp = kProducerWarp + 1;
  constexpr int RW = C::kRows;
  constexpr int SLOTS = C::kSlots;
  constexpr uint32_t TILE = C::kTile;
  extern __shared__ __align__(1024) uint8_t smem[];

  if (smem_u32(smem) & 1023u) {  // 128-byte swizzle needs 1024-byte aligned tiles
    if (threadIdx.x == 0) record_status(kDevStatusBadSmemAlign, 100);
    return;
  }
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + C::kSub * TILE;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* bar_q = bars;
  uint64_t* bar_full = bars + 1;
  uint64_t* bar_empty = bars + 1 + SLOTS;
  uint64_t* bar_s = bars + 1 + 2 * SLOTS;  // [2] S_k ready
  uint64_t* bar_p = bar_s + 2;             // [2] P_k written (and O_k corrected)
  uint64_t* bar_o = bar_p + 2;             // [2] last P_k V done
  uint64_t* bar_drain = bar_o + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int N = p.N;
  const int Nk = p.Nk;
  const int ntk = (Nk + 127) >> 7;  // key tiles
  // Heaviest query blocks first (they see the most keys under the causal
  // mask), a few heads at a time; the key ranges of one block side by side.
  int rank, bh;
  grouped_order(static_cast<int>(blockIdx.x), p.nblocks * p.splits, p.BH, p.head_group, rank, bh);
  const int qb = p.nblocks - 1 - rank / p.splits;
  const int split = rank % p.splits;
  const int j0 = split * p.tps;  // first key tile of this CTA's range
  // n_sub[k]: key tiles of this range that sub-tile k sees (all tiles up to
  // the one holding the last visible key of its last row, within the range)
  int n_sub[2];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int row0 = qb * RW + k * 128;
    int n = 0;
    if (k < C::kSub && row0 < N) {
      const int last = min(row0 + 127, N - 1);
      n = p.causal ? min(ntk, (last + p.q_off) / 128 + 1) : ntk;
    }
    n_sub[k] = max(0, min(n - j0, p.tps));
  }
  const int nmax = max(n_sub[0], n_sub[1]);

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < SLOTS; ++s) {
      mbar_init(&bar_full[s], 1);
      mbar_init(&bar_empty[s], 1);
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(&bar_s[k], 1);
      mbar_init(&bar_p[k], 128);
      mbar_init(&bar_o[k], 1);
    }
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint64_t tmo = p.timeout_ns;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && nmax > 0) {
      prefetch_tensormap(&p.tm_q);
      prefetch_tensormap(&p.tm_k);
      prefetch_tensormap(&p.tm_v);
      mbar_arrive_expect_tx(bar_q, TILE * (n_sub[1] > 0 ? 2u : 1u));
#pragma unroll
      for (int c = 0; c < C::kChunks; ++c) {
        tma_load_3d(sQ + c * 16384, &p.tm_q, bar_q, c * C::kChunkElems, qb * RW, bh);
        if (n_sub[1] > 0)
          tma_load_3d(sQ + TILE + c * 16384, &p.tm_q, bar_q, c * C::kChunkElems, qb * RW + 128, bh);
      }
      int last_par[SLOTS];
#pragma unroll
      for (int s = 0; s < SLOTS; ++s) last_par[s] = -1;
      bool ok = true;
      for (int j = 0; j < nmax && ok; ++j) {
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          const int idx = 2 * j + x;
          const int slot = idx % SLOTS;
          const uint32_t ph = (idx / SLOTS) & 1;
          if (!mbar_wait(&bar_empty[slot], ph ^ 1u, abort_flag, tmo, 101)) {
            ok = false;
            break;
          }
          if (idx == 0 && (p.debug_flags & kDebugSkipFirstKV)) continue;  // injected stall
          mbar_arrive_expect_tx(&bar_full[slot], TILE);
          const CUtensorMap* m = x ? &p.tm_v : &p.tm_k;
#pragma unroll
          for (int c = 0; c < C::kChunks; ++c)
            tma_load_3d(sKV + slot * TILE + c * 16384, m, &bar_full[slot], c * C::kChunkElems, (j0 + j) * 128, bh);
#pragma unroll
          for (int s = 0; s < SLOTS; ++s)
            if (s == slot) last_par[s] = static_cast<int>(ph);
        }
      }
      // Let every copy issued so far land before the CTA can exit (on the
      // normal path these phases have long completed; after an abort by any
      // role some may still be in flight).
      {
        drain_wait(bar_q, 0, 102);
#pragma unroll
        for (int s = 0; s < SLOTS; ++s)
          if (last_par[s] >= 0) drain_wait(&bar_full[s], static_cast<uint32_t>(last_par[s]), 103);
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && nmax > 0) {
      constexpr uint32_t idesc_s = idesc_16_f32(E::kMmaFmt, 128, 128, 0, 0);  // Q, K both K-major
      constexpr uint32_t idesc_o = idesc_16_f32(E::kMmaFmt, 128, D, 0, 1);    // P from TMEM, V MN-major
      const uint32_t sq0 = smem_u32(sQ);
      const uint32_t skv0 = smem_u32(sKV);
      auto kslot = [&](int j) { return (2 * j) % SLOTS; };
      auto kph = [&](int j) { return static_cast<uint32_t>(((2 * j) / SLOTS) & 1); };
      auto vslot = [&](int j) { return (2 * j + 1) % SLOTS; };
      auto vph = [&](int j) { return static_cast<uint32_t>(((2 * j + 1) / SLOTS) & 1); };
      // K-major view (Q, K) and MN-major view (V) of the tiles, built once
      const SmemDesc dK = make_desc_sw128(sq0, 16, 1024);
      const SmemDesc dMN = make_desc_sw128(skv0, 16384, 1024);
      auto issue_s = [&](int k, int slot) {
        const uint32_t a0 = k * TILE;                   // Q_k, relative to sQ
        const uint32_t b0 = (skv0 - sq0) + slot * TILE;  // K_j, relative to sQ
        const uint32_t dt = tmem + k * 256;
#pragma unroll
        for (int kk = 0; kk < C::kSSteps; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;  // 32 bytes of each row per MMA
          if constexpr (E::kF8)
            mma_ss_f8(dt, desc_at(dK, a0 + off), desc_at(dK, b0 + off), idesc_s, kk > 0 ? 1u : 0u);
          else
            mma_ss(dt, desc_at(dK, a0 + off), desc_at(dK, b0 + off), idesc_s, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int k, int slot, bool acc) {
        const uint32_t b0 = slot * TILE;  // V_j, relative to the ring
        const uint32_t dt = tmem + k * 256 + 128;
        const uint32_t at = tmem + k * 256;
        // each MMA takes kKStep keys: 8 TMEM columns of P, kKStep 128-byte rows of V
#pragma unroll
        for (int kk = 0; kk < C::kPVSteps; ++kk) {
          if constexpr (E::kF8)
            mma_ts_f8(dt, at + kk * 8, desc_at(dMN, b0 + kk * C::kKStep * 128), idesc_o, (acc || kk > 0) ? 1u : 0u);
          else
            mma_ts(dt, at + kk * 8, desc_at(dMN, b0 + kk * C::kKStep * 128), idesc_o, (acc || kk > 0) ? 1u : 0u);
        }
      };
      const int n0 = n_sub[0], n1 = n_sub[1];
      bool ok = mbar_wait(bar_q, 0, abort_flag, tmo, 110);
      ok = ok && mbar_wait(&bar_full[kslot(0)], kph(0), abort_flag, tmo, 111);
      if (ok) {
        tc_fence_after();
        if (n0 > 0) {
          issue_s(0, kslot(0));
          tc_commit(&bar_s[0]);
        }
        if (n1 > 0) {
          issue_s(1, kslot(0));
          tc_commit(&bar_s[1]);
        }
        tc_commit(&bar_empty[kslot(0)]);
      }
      for (int j = 0; j < nmax && ok; ++j) {
        const bool knext = (j + 1 < nmax);
        // V_j and K_(j+1) have long landed by now; their waits come before the
        // wait for P_0(j), so that no barrier wait sits between P_0 V_j and
        // S_0(j+1) on sub-tile 0's critical path
        if (!mbar_wait(&bar_full[vslot(j)], vph(j), abort_flag, tmo, 112)) break;
        if (knext && !mbar_wait(&bar_full[kslot(j + 1)], kph(j + 1), abort_flag, tmo, 114)) break;
        tc_fence_after();
        if (j < n0) {
          if (!mbar_wait(&bar_p[0], j & 1, abort_flag, tmo, 113)) break;
          tc_fence_after();
          issue_pv(0, vslot(j), j > 0);
          if (j == n0 - 1) tc_commit(&bar_o[0]);
        }
        if (j + 1 < n0) {
          issue_s(0, kslot(j + 1));
          tc_commit(&bar_s[0]);
        }
        if (j < n1) {
          if (!mbar_wait(&bar_p[1], j & 1, abort_flag, tmo, 115)) break;
          tc_fence_after();
          issue_pv(1, vslot(j), j > 0);
          if (j == n1 - 1) tc_commit(&bar_o[1]);
        }
        tc_commit(&bar_empty[vslot(j)]);
        if (j + 1 < n1) {
          issue_s(1, kslot(j + 1));
          tc_commit(&bar_s[1]);
        }
        if (knext) tc_commit(&bar_empty[kslot(j + 1)]);
      }
      // All MMAs issued by this thread must be complete before TMEM is freed.
      tc_commit(bar_drain);
      drain_wait(bar_drain, 0, 116);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    const int wq = warp & 3;  // TMEM lane quadrant
    const int row = wq * 32 + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const float c = p.scale_log2;
    // The reference max moves only if exps would exceed 2^kLazy.  For e4m3
    // probabilities the limit is 2^2 and every P is scaled by 2^6 before it
    // is rounded, so that P stays in [0, 256] (inside e4m3's range, 448) and
    // all but negligible probabilities keep e4m3's full 3-bit precision
    // instead of falling to its subnormals; l carries the same factor, which
    // cancels in O / l and is taken out of the LSE.
    constexpr float kLazy = E::kF8 ? 2.0f : 8.0f;
    constexpr float kPLog2 = E::kF8 ? 6.0f : 0.0f;
    const float thr = kLazy / c;

    // One step of the online softmax for sub-tile k, key tile j: load S_k,
    // mask, move the reference maximum if needed (rescaling O_k), write P_k
    // as bf16 over S_k and signal the MMA issuer.  Returns false if a wait
    // gave up (the outcome is warp-uniform: the tcgen05.ld/st are
    // warp-collective).
    auto step = [&](int k, int j, float& m_ref, float& l) -> bool {
      const uint32_t tS = lane_base + k * 256;
      const uint32_t tO = tS + 128;
      if (!__all_sync(0xffffffffu, mbar_wait(&bar_s[k], j & 1, abort_flag, tmo, 120 + k))) return false;
      tc_fence_after();
      uint32_t sr[128];
      tmem_ld32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tmem_ld32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[64]));
      tmem_ld32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(&sr[96]));
      tmem_wait_ld();
      const int key0 = (j0 + j) * 128;
      const int q_row = qb * RW + k * 128 + row;
      // masking is needed where the sub-tile's first row does not see the
      // whole tile, or on the ragged last key tile
      const bool part = p.causal && key0 + 127 > qb * RW + k * 128 + p.q_off;
      if (part || key0 + 128 > Nk) {
        const int lim = min(part ? q_row + p.q_off - key0 : 127, Nk - 1 - key0);  // last visible column
#pragma unroll
        for (int i = 0; i < 128; ++i)
          if (i > lim) sr[i] = __float_as_uint(-INFINITY);
      }
      // row maximum: eight independent chains of 3-input max
      float mxa[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) mxa[t] = __uint_as_float(sr[t]);
#pragma unroll
      for (int i = 8; i < 128; i += 2)
        mxa[(i >> 1) & 7] = max3f(mxa[(i >> 1) & 7], __uint_as_float(sr[i]), __uint_as_float(sr[i + 1]));
      const float mx = fmaxf(max3f(mxa[0], mxa[1], mxa[2]), max3f(mxa[3], mxa[4], max3f(mxa[5], mxa[6], mxa[7])));
      const float m_new = (mx > m_ref + thr) ? mx : m_ref;
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      const float alpha = ex2((m_ref - m_use) * c);
      const uint64_t c2 = f2_pack(c, c);
      const uint64_t neg2 = f2_pack(kPLog2 - m_use * c, kPLog2 - m_use * c);
      uint64_t suma[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
      uint32_t pk[64];  // 16-bit: one pair of keys per word; e4m3: words 0..31, four keys each
      uint64_t pk2_prev = 0;  // e4m3: the even pair, held until the odd one completes a word
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        const uint64_t x = f2_fma(f2_pack(__uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1])), c2, neg2);
        uint64_t pp;
        if ((i & 7) >= 8 - kEmuPairs) {  // kEmuPairs of every 8 pairs on the FMA pipe
          pp = ex2_fma2(x);
        } else {
          float x0, x1;
          f2_unpack(x, x0, x1);
          pp = f2_pack(ex2(x0), ex2(x1));
        }
        suma[i & 1] = f2_add(suma[i & 1], pp);
        float p0, p1;
        f2_unpack(pp, p0, p1);
        if constexpr (E::kF8) {
          if (i & 1) {
            float q0, q1;
            f2_unpack(pk2_prev, q0, q1);
            pk[i >> 1] = E::pack4(q0, q1, p0, p1);
          } else {
            pk2_prev = pp;
          }
        } else {
          pk[i] = E::pack2(p0, p1);
        }
      }
      float s0, s1, s2, s3;
      f2_unpack(suma[0], s0, s1);
      f2_unpack(suma[1], s2, s3);
      l = l * alpha + ((s0 + s1) + (s2 + s3));
#pragma unroll
      for (int i = 0; i < C::kPCols / 16; ++i)
        tmem_st16(tS + 16 * i, *reinterpret_cast<const uint32_t(*)[16]>(&pk[16 * i]));
      if (j > 0 && __any_sync(0xffffffffu, alpha != 1.0f)) {
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[32];
          tmem_ld32(tO + 32 * cc, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(tO + 32 * cc, o);
        }
      }
      m_ref = m_new;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bar_p[k]);
      return true;
    };

    // Epilogue of sub-tile k once its last P V product is done: O = O / l
    // as bf16, LSE = m scale + ln l.
    auto epilogue = [&](int k, float m_ref, float l) {
      if (!__all_sync(0xffffffffu, mbar_wait(&bar_o[k], 0, abort_flag, tmo, 122 + k))) return;
      tc_fence_after();
      const uint32_t tO = lane_base + k * 256 + 128;
      const int q_row = qb * RW + k * 128 + row;
      if (p.part_o != nullptr) {
        // one key range of a split row: O normalised by this range's own sum,
        // and the range's logsumexp (-inf if the row saw none of its keys)
        const float inv_l = l > 0.f ? p.o_mul / l : 0.f;
        const size_t prow = (static_cast<size_t>(bh) * p.splits + split) * N + q_row;
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[32];
          tmem_ld32(tO + 32 * cc, o);
          tmem_wait_ld();
          if (q_row < N) {
            float4* dst = reinterpret_cast<float4*>(p.part_o + prow * D + 32 * cc);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              dst[i] = make_float4(__uint_as_float(o[4 * i]) * inv_l, __uint_as_float(o[4 * i + 1]) * inv_l,
                                   __uint_as_float(o[4 * i + 2]) * inv_l, __uint_as_float(o[4 * i + 3]) * inv_l);
          }
        }
        if (q_row < N) p.part_lse[prow] = l > 0.f ? m_ref * p.scale + __logf(l) - kPLog2 * 0.6931471805599453f : -INFINITY;
        return;
      }
      const float inv_l = p.o_mul / l;
      TO* orow = static_cast<TO*>(p.o) + (static_cast<size_t>(bh) * N + q_row) * D;
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t o[32];
        tmem_ld32(tO + 32 * cc, o);
        tmem_wait_ld();
        if (q_row < N) {
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            w[i] = Elem<TO>::pack2(__uint_as_float(o[2 * i]) * inv_l, __uint_as_float(o[2 * i + 1]) * inv_l);
          uint4* dst = reinterpret_cast<uint4*>(orow + 32 * cc);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
        }
      }
      if (q_row < N)
        p.lse[static_cast<size_t>(bh) * N + q_row] = m_ref * p.scale + __logf(l) - kPLog2 * 0.6931471805599453f;
    };

    const int k = warp >> 2;  // sub-tile
    const int n = k ? n_sub[1] : n_sub[0];
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n && ok; ++j) ok = step(k, j, m_ref, l);
    if (ok && n > 0) epilogue(k, m_ref, l);
    if (n == 0 && p.part_o != nullptr) {
      // a range that holds none of this sub-tile's visible keys: an empty part
      const int q_row = qb * RW + k * 128 + row;
      if (q_row < N) {
        const size_t prow = (static_cast<size_t>(bh) * p.splits + split) * N + q_row;
        float4* dst = reinterpret_cast<float4*>(p.part_o + prow * D);
#pragma unroll
        for (int i = 0; i < D / 4; ++i) dst[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        p.part_lse[prow] = -INFINITY;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, C::kTmemCols);
}

}  // namespace exattn

namespace exattn {

// Combines the key ranges of a split forward: per query row,
//   LSE = log sum_s exp(LSE_s),  O = sum_s exp(LSE_s - LSE) O_s,
// the merge of online-softmax partial results ("11.11 Flash Attention",
// section "Flash Attention: The Key Insight": partial maxima and sums of
// blocks combine exactly).  One warp per row; each lane holds d / 32 columns.
template <int D, typename T>
__global__ void __launch_bounds__(256) attn_fwd_merge_kernel(const float* __restrict__ part_o,
                                                             const float* __restrict__ part_lse,
                                                             void* __restrict__ o, float* __restrict__ lse, int BH,
                                                             int N, int splits) {
  constexpr int V = D / 32;  // columns per lane
  const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);  // over BH * N
  const int lane = threadIdx.x & 31;
  if (row >= static_cast<long long>(BH) * N) return;
  const long long bh = row / N, i = row - bh * N;
  float m = -INFINITY;
  for (int s = 0; s < splits; ++s) m = fmaxf(m, part_lse[(bh * splits + s) * N + i]);
  float acc[V];
#pragma unroll
  for (int c = 0; c < V; ++c) acc[c] = 0.f;
  float wsum = 0.f;
  if (m != -INFINITY) {
    for (int s = 0; s < splits; ++s) {
      const long long pr = (bh * splits + s) * N + i;
      const float w = __expf(part_lse[pr] - m);
      wsum += w;
      const float* src = part_o + pr * D + lane * V;
      if constexpr (V >= 4) {
#pragma unroll
        for (int c4 = 0; c4 < V / 4; ++c4) {
          const float4 x = reinterpret_cast<const float4*>(src)[c4];
          acc[4 * c4] += w * x.x;
          acc[4 * c4 + 1] += w * x.y;
          acc[4 * c4 + 2] += w * x.z;
          acc[4 * c4 + 3] += w * x.w;
        }
      } else {
        const float2 x = *reinterpret_cast<const float2*>(src);
        acc[0] += w * x.x;
        acc[1] += w * x.y;
      }
    }
  }
  const float inv = wsum > 0.f ? 1.0f / wsum : 0.f;
  uint32_t w2[V / 2];
#pragma unroll
  for (int c = 0; c < V / 2; ++c) w2[c] = Elem<T>::pack2(acc[2 * c] * inv, acc[2 * c + 1] * inv);
  T* dst = static_cast<T*>(o) + row * D + lane * V;
  if constexpr (V == 8)
    *reinterpret_cast<uint4*>(dst) = make_uint4(w2[0], w2[1], w2[2], w2[3]);
  else if constexpr (V == 4)
    *reinterpret_cast<uint2*>(dst) = make_uint2(w2[0], w2[1]);
  else
    *reinterpret_cast<uint32_t*>(dst) = w2[0];
  if (lane == 0) lse[row] = (m == -INFINITY) ? -INFINITY : m + __logf(wsum);
}

}  // namespace exattn

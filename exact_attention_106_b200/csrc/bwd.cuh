// Backward kernels.  The forward keeps only Q, K, V, O and the per-row
// logsumexp; the backward recomputes the probabilities tile by tile from them
// ("Walk through the FlashAttention algorithm ...", answer to "How does the
// backward pass avoid storing the n x n attention matrix?"; "11.11 Flash
// Attention", section "The Recomputation Trade-off").  The gradient formulas
// are the chain rule of O = softmax(scale Q K^T) V (the pages give none):
//   dV = P^T dO,  dP = dO V^T,  D = rowsum(dO o O),  dS = P o (dP - D),
//   dQ = scale dS K,  dK = scale dS^T Q.
//
// Stage 1 (attn_bwd_preprocess_kernel): D and LSE*log2(e) per row into a
//   padded workspace; zero the fp32 dQ accumulator.
// Stage 2 (attn_bwd_kernel): one CTA per (batch, head, 128-key tile j).  It
//   keeps K_j, V_j in shared memory and dK_j, dV_j in tensor memory, and walks
//   the query tiles i (i >= j under the causal mask).  Per query tile:
//     S^T = K_j Q_i^T            (tcgen05, TMEM)
//     P^T = exp2(S^T c - LSE_i)  (registers -> TMEM as 16-bit, over S^T)
//     dP^T = V_j dO_i^T          (tcgen05, TMEM)
//     dV_j += P^T dO_i           (A operand read from TMEM)
//     dS^T = P^T o (dP^T - D_i)  (registers -> shared memory as 16-bit)
//     dK_j += dS^T Q_i ;  dQ_i-partial = dS K_j  (tcgen05)
//   and adds the dQ partial into the fp32 accumulator: four drain warps read
//   it from tensor memory (handing the columns back at once), stage it in
//   shared memory and let the TMA engine add it into global memory.
// Stage 3 (attn_bwd_dq_convert_kernel): dQ = T(scale * accumulator), T the element type
// (bf16 or fp16; inputs, gradients, P and dS all use it).
#pragma once
#include "ptx.cuh"

namespace exattn {

struct BwdParams {
  CUtensorMap tm_q;  // 3-D {d, N, B*H}, box {64, 128, 1}, 128-byte swizzle
  CUtensorMap tm_k;
  CUtensorMap tm_v;
  CUtensorMap tm_do;
  CUtensorMap tm_dq;  // fp32 2-D {d, B*H*Np}, box {32, 32}, 128-byte swizzle (dQ accumulator)
  void* dk;  // [B*H, N, d] of the element type T
  void* dv;
  float* dq_acc;       // [BH, Np, d]
  const float* dvec;   // [BH, Np]  D
  const float* lse2;   // [BH, Np]  LSE * log2(e), +inf on padded rows
  int N;
  int Np;
  int BH;
  int ntiles;  // ceil(N / 128)
  int head_group;  // heads whose CTAs are scheduled together (L2 reuse of Q/dO/dQ)
  int causal;
  int paired;      // causal items taken in pairs (j, ntiles - 1 - j); see the kernel
  float scale;
  float scale_log2;
  unsigned long long timeout_ns;
  unsigned int debug_flags;
};

template <int D>
struct BwdCfg {
  // warps 0..3: compute, query columns 0..63; warps 4..7: columns 64..127;
  // warps 8..11: dQ drain; warp 12: TMA producer; warp 13: MMA issuer of
  // the products that follow the scores (S^T, dP^T, dV); warp 14: MMA issuer
  // of the products of dS (dQ, dK); warp 15: idle (completes the warpgroup).
  static constexpr int kThreads = 512;
  // Registers per thread: the launch gives every thread R (the compiled count,
  // at most 65536 / 512 = 128).  Warpgroup 3 (producer, MMA, idle) drops to
  // kRegsSide and the drain warpgroup rises to kRegsDrain, so that it can hold
  // a whole 128-column dQ partial.  This fits if kRegsDrain - R <= R - kRegsSide,
  // i.e. R >= kRegsMin; the host refuses to launch a build with fewer.
  static constexpr int kRegsDrain = 168;
  static constexpr int kRegsSide = 80;
  static constexpr int kRegsMin = (kRegsDrain + kRegsSide + 1) / 2;
  static constexpr int kRegsMax = 65536 / kThreads;
  static_assert(kRegsMin <= kRegsMax, "register split cannot fit");
  // per sub-partition: one warp of each warpgroup
  static_assert(2 * kRegsMax + kRegsDrain + kRegsSide <= 512, "sub-partition register file");
  static constexpr uint32_t kTile = 128u * D * 2u;
  static constexpr int kChunks = D / 64;
  static constexpr uint32_t kOffK = 0;
  static constexpr uint32_t kOffV = kTile;
  static constexpr uint32_t kOffQ = 2 * kTile;   // 2 stages
  static constexpr uint32_t kOffDO = 4 * kTile;  // 2 stages
  static constexpr uint32_t kOffDS = 6 * kTile;  // 128 x 128 16-bit
  static constexpr uint32_t kOffVec = kOffDS + 32768;  // 2 stages x (LSE2[128], D[128]) fp32
  // dQ staging: at d = 128 the dO buffer of the step being drained (dead once
  // dV and dP have read it); at d = 64 a buffer of its own (32 KB).
  static constexpr uint32_t kOffStage = kOffVec + 2048;
  static constexpr uint32_t kStageBytes = (D == 128) ? 0u : 32768u;
  static constexpr uint32_t kOffBar = kOffStage + kStageBytes;
  static constexpr uint32_t kSmem = kOffBar + 256;
  // tensor-memory columns
  static constexpr uint32_t kColDK = 0;
  static constexpr uint32_t kColDV = D;
  static constexpr uint32_t kColS = 2 * D;
  static constexpr uint32_t kColDP = 2 * D + 128;
  static constexpr uint32_t kColDQ = (D == 128) ? kColDP : 384;  // d=128: dQ reuses dP's columns
};

// X[128 x 128] = A[128 x D] B[128 x D]^T with both operands K-major D-wide
// tiles at offsets a0, b0 from the shared-memory base (S^T and dP^T).
template <int D, typename T>
__device__ __forceinline__ void bwd_issue_t(uint32_t d_tmem, SmemDesc dKm, uint32_t a0, uint32_t b0) {
  constexpr uint32_t idesc = idesc_16_f32(Elem<T>::kMmaFmt, 128, 128, 0, 0);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
    mma_ss(d_tmem, desc_at(dKm, a0 + off), desc_at(dKm, b0 + off), idesc, kk > 0 ? 1u : 0u);
  }
}

// T: the 16-bit element type of Q, K, V, dO and the gradients.
// kPersist: the CTA walks several work units (see below); otherwise it runs
// the single unit blockIdx.x, and the step and item counters fold to their
// first values at compile time.
template <int D, typename T, bool kPersist>
__global__ void __launch_bounds__(512, 1) attn_bwd_kernel(const __grid_constant__ BwdParams p) {
  using C = BwdCfg<D>;
  using E = Elem<T>;
  constexpr int kProducerWarp = 12;
  constexpr int kMmaWarp = 13;   // also allocates TMEM
  constexpr int kMmaWarp2 = 14;
  constexpr uint32_t TILE = C::kTile;
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) record_status(kDevStatusBadSmemAlign, 200);
    return;
  }
  uint8_t* sK = smem + C::kOffK;
  uint8_t* sV = smem + C::kOffV;
  uint8_t* sQ = smem + C::kOffQ;
  uint8_t* sDO = smem + C::kOffDO;
  uint8_t* sDS = smem + C::kOffDS;
  float* sVec = reinterpret_cast<float*>(smem + C::kOffVec);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* bar_kv = bars + 0;
  uint64_t* bar_qfull = bars + 1;    // [2] Q_i, LSE_i, D_i landed
  uint64_t* bar_qempty = bars + 3;   // [2] Q_i, LSE_i, D_i consumed (MMA commit after dK)
  uint64_t* bar_dofull = bars + 5;   // [2] dO_i landed
  uint64_t* bar_doempty = bars + 7;  // [2] dO_i buffer free (the drain warps, after their staging; 4 arrivals)
  uint64_t* bar_s = bars + 9;        // S^T ready
  uint64_t* bar_dp = bars + 10;      // dP^T ready
  uint64_t* bar_p = bars + 11;       // P^T written (256 arrivals)
  uint64_t* bar_ds = bars + 12;      // dS written to smem (256 arrivals)
  uint64_t* bar_dsfree = bars + 13;  // dS consumed by the dQ and dK MMAs
  uint64_t* bar_dqfull = bars + 14;  // dQ partial ready in TMEM
  uint64_t* bar_dqfree = bars + 15;  // dQ partial read out of TMEM (128 arrivals)
  uint64_t* bar_final = bars + 16;   // all MMAs done (one commit from each issuer)
  uint64_t* bar_drain = bars + 17;   // both issuers' MMAs done (2 commits)
  // [2] dV_i done, so dO_i is read (issuer commit), one per dO stage: the
  // drain of step i waits on stage i % 2, whose next phase needs dO_(i+2),
  // which only loads after that drain has released the stage, so the
  // barrier can never run two phases ahead of its waiter
  uint64_t* bar_dvdone = bars + 18;
  uint64_t* bar_accfree = bars + 20;  // dK, dV of an item read out by the epilogue (256 arrivals)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 21);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int N = p.N;
  const int ntq = p.ntiles;  // query tiles
  // Work units.  With kPersist false the CTA runs the single item blockIdx.x
  // (key tile j, head bh), and the hardware hands out the items as SMs free
  // up: key tile 0 first (under the causal mask it sees the most query
  // tiles), a few heads at a time.  With kPersist (short rows, where a CTA's
  // start-up and epilogue weigh) one CTA per SM walks the units blockIdx.x,
  // blockIdx.x + gridDim.x, ...; under the causal mask (p.paired) a unit is
  // the pair of key tiles (j, ntq - 1 - j) of one head, heavier first, which
  // together see ntq + 1 query tiles, so that a fixed stride over equal units
  // balances the SMs as well as the hardware's scheduling would (with an odd
  // ntq the middle tile stands alone, last in its head's order).  Every role
  // walks the same sequence; a step's rings and barriers take their phases
  // from its index g in the CTA's whole sequence of steps (the counters are 0
  // without kPersist), so that one item's loads and products start while the
  // previous item's epilogue runs.
  const int npt = (ntq + 1) / 2;
  const bool paired = kPersist && p.causal && p.paired;
  constexpr int kHalves = kPersist ? 2 : 1;
  const int units = (paired ? npt : ntq) * p.BH;
  auto unit_item = [&](int u, int half, int& j, int& bh, int& i0, int& n) -> bool {
    int r;
    grouped_order(u, paired ? npt : ntq, p.BH, p.head_group, r, bh);
    if (!paired) {
      j = r;
      i0 = p.causal ? j : 0;
      n = ntq - i0;  // >= 1
      return half == 0;
    }
    j = half ? ntq - 1 - r : r;
    i0 = j;
    n = ntq - j;  // >= 1
    return !(half && j == r);
  };

  if (threadIdx.x == 0) {
    mbar_init(bar_kv, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar_qfull[s], 1);
      mbar_init(&bar_qempty[s], 1);
      mbar_init(&bar_dofull[s], 1);
      mbar_init(&bar_doempty[s], 4);
    }
    mbar_init(bar_s, 1);
    mbar_init(bar_dp, 1);
    mbar_init(bar_p, 256);
    mbar_init(bar_ds, 256);
    mbar_init(bar_dsfree, 1);
    mbar_init(bar_dqfull, 1);
    mbar_init(bar_dqfree, 128);
    mbar_init(bar_final, 2);
    mbar_init(bar_drain, 2);
    mbar_init(&bar_dvdone[0], 1);
    mbar_init(&bar_dvdone[1], 1);
    mbar_init(bar_accfree, 256);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint64_t tmo = p.timeout_ns;

  if (warp >= 12) {
  setmaxnreg_dec<C::kRegsSide>();
  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&p.tm_q);
      prefetch_tensormap(&p.tm_k);
      prefetch_tensormap(&p.tm_v);
      prefetch_tensormap(&p.tm_do);
      int lq[2] = {-1, -1}, ld[2] = {-1, -1};  // parity of the last loads into each stage
      int lkv = -1;                            // parity of the last K, V load
      bool ok = true;
      int g0_ = 0, t_ = 0;  // first step of the item, items done
      for (int wu = blockIdx.x; wu < units && ok; wu += kPersist ? static_cast<int>(gridDim.x) : units)
      for (int half = 0; half < kHalves && ok; ++half) {
        int j, bh, i0, n;
        if (!unit_item(wu, half, j, bh, i0, n)) continue;
        const int g0 = kPersist ? g0_ : 0;  // this item's first step
        const int t = kPersist ? t_ : 0;    // items before this one
        auto load_kv = [&]() {
          if (t > 0 || !(p.debug_flags & kDebugSkipFirstKV)) {  // else: injected stall
            mbar_arrive_expect_tx(bar_kv, 2 * TILE);
#pragma unroll
            for (int c = 0; c < C::kChunks; ++c) {
              tma_load_3d(sK + c * 16384, &p.tm_k, bar_kv, c * 64, j * 128, bh);
              tma_load_3d(sV + c * 16384, &p.tm_v, bar_kv, c * 64, j * 128, bh);
            }
            lkv = t & 1;
          }
        };
        if (t == 0) load_kv();  // a fresh CTA: K and V first, the first S^T needs K at once
        for (int it = 0; it < n; ++it) {
          const int g = g0 + it;
          const int st = g & 1;
          const uint32_t ph = (g >> 1) & 1;
          const int i = i0 + it;
          if (!mbar_wait(&bar_qempty[st], ph ^ 1u, abort_flag, tmo, 201)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bar_qfull[st], TILE + 1024);
#pragma unroll
          for (int c = 0; c < C::kChunks; ++c)
            tma_load_3d(sQ + st * TILE + c * 16384, &p.tm_q, &bar_qfull[st], c * 64, i * 128, bh);
          const size_t vrow = static_cast<size_t>(bh) * p.Np + static_cast<size_t>(i) * 128;
          bulk_load(sVec + st * 256, p.lse2 + vrow, 512, &bar_qfull[st]);
          bulk_load(sVec + st * 256 + 128, p.dvec + vrow, 512, &bar_qfull[st]);
          if (st == 0) lq[0] = static_cast<int>(ph); else lq[1] = static_cast<int>(ph);
          if (!mbar_wait(&bar_doempty[st], ph ^ 1u, abort_flag, tmo, 202)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bar_dofull[st], TILE);
#pragma unroll
          for (int c = 0; c < C::kChunks; ++c)
            tma_load_3d(sDO + st * TILE + c * 16384, &p.tm_do, &bar_dofull[st], c * 64, i * 128, bh);
          if (st == 0) ld[0] = static_cast<int>(ph); else ld[1] = static_cast<int>(ph);
          if (it == 0 && t > 0) {
            // A later item's K_j, V_j, after its first Q and dO, once every
            // product of the previous item that reads K or V is done: S^T and
            // dP^T (the last dP^T commit covers the S^T before it) and dQ of
            // its last step g0 - 1.  dK and dV read neither, so the load
            // overlaps them and the item's epilogue.  The two barriers cannot
            // be a phase further on: this item's dP^T and dQ need the K and V
            // loaded here.
            if (!(mbar_wait(bar_dp, (g0 - 1) & 1, abort_flag, tmo, 206) &&
                  mbar_wait(bar_dqfull, (g0 - 1) & 1, abort_flag, tmo, 227))) {
              ok = false;
              break;
            }
            load_kv();
          }
        }
        g0_ += n;
        ++t_;
      }
      // Let every copy issued so far land before the CTA can exit.
      if (lkv >= 0) drain_wait(bar_kv, static_cast<uint32_t>(lkv), 203);
      for (int s = 0; s < 2; ++s) {
        if (lq[s] >= 0) drain_wait(&bar_qfull[s], static_cast<uint32_t>(lq[s]), 204);
        if (ld[s] >= 0) drain_wait(&bar_dofull[s], static_cast<uint32_t>(ld[s]), 205);
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp || warp == kMmaWarp2) {
    // ------------------------------------------------------------ MMA issuers
    // Two threads issue MMAs into the one tensor pipe, each waiting only on
    // its own inputs, so that one keeps the pipe busy while the other waits.
    // A commit covers only its own thread's MMAs; every hand-off between
    // the two goes through a barrier below.
    if (lane == 0) {
      constexpr uint32_t idesc_kv = idesc_16_f32(E::kMmaFmt, 128, D, 0, 1);  // dV, dK: B = dO / Q MN-major
      constexpr uint32_t idesc_q = idesc_16_f32(E::kMmaFmt, 128, D, 1, 1);   // dQ: A = dS MN-major, B = K MN-major
      // K-major and MN-major views of this CTA's shared memory, built once;
      // every operand below is an offset from the dynamic shared-memory base.
      const SmemDesc dKm = make_desc_sw128(smem_u32(smem), 16, 1024);
      const SmemDesc dMN = make_desc_sw128(smem_u32(smem), 16384, 1024);
      constexpr uint32_t oK = C::kOffK, oV = C::kOffV, oQ = C::kOffQ, oDO = C::kOffDO, oDS = C::kOffDS;
      if (warp == kMmaWarp) {
        // S^T = K Q_i^T, dP^T = V dO_i^T, dV += P^T dO_i
        bool ok = true;
        int g0_ = 0, t_ = 0;
        for (int wu = blockIdx.x; wu < units && ok; wu += kPersist ? static_cast<int>(gridDim.x) : units)
        for (int half = 0; half < kHalves && ok; ++half) {
          int j, bh, i0, n;
          if (!unit_item(wu, half, j, bh, i0, n)) continue;
          const int g0 = kPersist ? g0_ : 0;  // this item's first step
          const int t = kPersist ? t_ : 0;    // items before this one
          const int st0 = g0 & 1;
          const uint32_t ph0 = (g0 >> 1) & 1;
          ok = mbar_wait(bar_kv, t & 1, abort_flag, tmo, 210) && mbar_wait(&bar_qfull[st0], ph0, abort_flag, tmo, 211);
          if (!ok) break;
          tc_fence_after();
          bwd_issue_t<D, T>(tmem + C::kColS, dKm, oK, oQ + st0 * TILE);
          tc_commit(bar_s);
          // dP^T overwrites the previous step's dP^T, read once its dS is
          // written, and at d = 128 also that step's dQ partial
          if (g0 > 0) {
            ok = mbar_wait(bar_ds, (g0 - 1) & 1, abort_flag, tmo, 207) &&
                 (D != 128 || mbar_wait(bar_dqfree, (g0 - 1) & 1, abort_flag, tmo, 208));
            if (!ok) break;
          }
          ok = mbar_wait(&bar_dofull[st0], ph0, abort_flag, tmo, 212);
          if (!ok) break;
          tc_fence_after();
          bwd_issue_t<D, T>(tmem + C::kColDP, dKm, oV, oDO + st0 * TILE);
          tc_commit(bar_dp);
          for (int it = 0; it < n; ++it) {
            const int g = g0 + it;
            const int st = g & 1;
            const int st1 = (g + 1) & 1;
            const uint32_t ph1 = ((g + 1) >> 1) & 1;
            // dV += P^T dO_i   (A = P^T from TMEM, K = 128 queries; queries 0..63
            // sit in columns [0,32) of the score block, 64..127 in [64,96)); the
            // item's first dV starts over once the previous item's dV is read out
            if (!mbar_wait(bar_p, g & 1, abort_flag, tmo, 213) ||
                (it == 0 && t > 0 && !mbar_wait(bar_accfree, (t - 1) & 1, abort_flag, tmo, 209))) {
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_ts(tmem + C::kColDV, tmem + C::kColS + (kk >> 2) * 64 + (kk & 3) * 8,
                     desc_at(dMN, oDO + st * TILE + kk * 2048), idesc_kv, (it > 0 || kk > 0) ? 1u : 0u);
            tc_commit(&bar_dvdone[st]);  // also dP_i: both readers of dO_i are done
            if (it + 1 < n) {
              // next S^T as early as possible: its softmax overlaps dQ, dK of tile it
              if (!mbar_wait(&bar_qfull[st1], ph1, abort_flag, tmo, 214)) {
                ok = false;
                break;
              }
              tc_fence_after();
              bwd_issue_t<D, T>(tmem + C::kColS, dKm, oK, oQ + st1 * TILE);
              tc_commit(bar_s);
              // dP^T(it+1) overwrites dP^T(it), read once dS_i is written, and at
              // d = 128 also the dQ partial, free once the drain has read it
              if (!mbar_wait(bar_ds, g & 1, abort_flag, tmo, 215) ||
                  (D == 128 && !mbar_wait(bar_dqfree, g & 1, abort_flag, tmo, 217)) ||
                  !mbar_wait(&bar_dofull[st1], ph1, abort_flag, tmo, 218)) {
                ok = false;
                break;
              }
              tc_fence_after();
              bwd_issue_t<D, T>(tmem + C::kColDP, dKm, oV, oDO + st1 * TILE);
              tc_commit(bar_dp);
            }
          }
          if (!ok) break;
          tc_commit(bar_final);  // this issuer's products of the item are done
          g0_ += n;
          ++t_;
        }
      } else {
        // dQ_i partial = dS K_j, dK += dS^T Q_i
        bool ok = true;
        int g0_ = 0, t_ = 0;
        for (int wu = blockIdx.x; wu < units && ok; wu += kPersist ? static_cast<int>(gridDim.x) : units)
        for (int half = 0; half < kHalves && ok; ++half) {
          int j, bh, i0, n;
          if (!unit_item(wu, half, j, bh, i0, n)) continue;
          const int g0 = kPersist ? g0_ : 0;  // this item's first step
          const int t = kPersist ? t_ : 0;    // items before this one
          if (!mbar_wait(bar_kv, t & 1, abort_flag, tmo, 224)) {
            ok = false;
            break;
          }
          for (int it = 0; it < n; ++it) {
            const int g = g0 + it;
            const int st = g & 1;
            if (!mbar_wait(bar_ds, g & 1, abort_flag, tmo, 225)) {
              ok = false;
              break;
            }
            tc_fence_after();
            if (D != 128 && g > 0) {  // separate dQ columns: only the previous dQ must be drained
              if (!mbar_wait(bar_dqfree, (g - 1) & 1, abort_flag, tmo, 216)) {
                ok = false;
                break;
              }
              tc_fence_after();
            }
            // dQ first (A = dS MN-major in smem, B = K_j MN-major), so that its
            // drain overlaps dK
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_ss(tmem + C::kColDQ, desc_at(dMN, oDS + kk * 2048), desc_at(dMN, oK + kk * 2048), idesc_q,
                     kk > 0 ? 1u : 0u);
            tc_commit(bar_dqfull);
            // the item's first dK starts over once the previous item's dK is read out
            if (it == 0 && t > 0) {
              if (!mbar_wait(bar_accfree, (t - 1) & 1, abort_flag, tmo, 226)) {
                ok = false;
                break;
              }
              tc_fence_after();
            }
            // dK += dS^T Q_i   (A = dS^T K-major in smem, B = Q_i MN-major)
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t offa = (kk >> 2) * 16384 + (kk & 3) * 32;
              mma_ss(tmem + C::kColDK, desc_at(dKm, oDS + offa), desc_at(dMN, oQ + st * TILE + kk * 2048),
                     idesc_kv, (it > 0 || kk > 0) ? 1u : 0u);
            }
            tc_commit(bar_dsfree);
            tc_commit(&bar_qempty[st]);
          }
          if (!ok) break;
          tc_commit(bar_final);  // this issuer's products of the item are done
          g0_ += n;
          ++t_;
        }
      }
      tc_commit(bar_drain);
      drain_wait(bar_drain, 0, 219);
    }
    __syncwarp();
  }
  } else if (warp < 8) {
    // ------------------------------------------------------------ compute
    const int h = warp >> 2;  // query-column half
    const int wq = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    // Scores, dP and P are read and written in the 16-lane fragment layout:
    // thread t holds key rows 32wq + 16b + 8rr + t/4 (b, rr in {0, 1}) and, in
    // each 8-column group g of this half, the query pair 64h + 8g + 2(t%4) + {0, 1}.
    // A thread thus needs only 16 of the 64 LSE and D values of its half, and
    // each pair of them is one packed operand.
    const int g4 = lane >> 2, t4 = lane & 3;
    const uint32_t tS = tmem + lane_off + C::kColS + 64 * h;
    const uint32_t tDP = tmem + lane_off + C::kColDP + 64 * h;
    const float c = p.scale_log2;
    // dS tile: K-major, row = key, 128-byte swizzle (16-byte unit u of row k at
    // unit u ^ (k & 7)); stmatrix row address of this lane for block b, group g
    const uint32_t ds_lane = smem_u32(sDS) + h * 16384 + (32 * wq + (lane & 15)) * 128;
    const uint32_t ds_sw = lane & 7;
    bool ok = true;
    int g0_ = 0, t_ = 0;
    for (int wu = blockIdx.x; wu < units && ok; wu += kPersist ? static_cast<int>(gridDim.x) : units)
    for (int half = 0; half < kHalves && ok; ++half) {
    // only the step count and the padding bits stay live through the steps
    int n, pad = 0;  // pad bit 2b+rr: that key row is padding
    {
      int j, bh, i0;
      if (!unit_item(wu, half, j, bh, i0, n)) continue;
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (j * 128 + 32 * wq + 8 * q + g4 >= N) pad |= 1 << q;
    }
    const int g0 = kPersist ? g0_ : 0;  // this item's first step
    const int t = kPersist ? t_ : 0;    // items before this one
    for (int it = 0; it < n; ++it) {
      const int g = g0 + it;
      const int st = g & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(bar_s, g & 1, abort_flag, tmo, 220))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sr[2][32];
      tmem_ld16x256_x8(tS, sr[0]);
      tmem_ld16x256_x8(tS + (16u << 16), sr[1]);
      tmem_wait_ld();
      const float2* lse2 = reinterpret_cast<const float2*>(sVec + st * 256 + 64 * h + 2 * t4);
      const float2* dv2 = reinterpret_cast<const float2*>(sVec + st * 256 + 128 + 64 * h + 2 * t4);
      const bool diag = p.causal && (it == 0);
      // P^T = exp2(S^T c - LSE log2 e) in packed pairs; kEmuPairs of every 8
      // pairs on the FMA pipe (ex2_fma2), the rest on the special-function unit
      const uint64_t c2 = f2_pack(c, c);
      uint64_t pf[2][16];  // [b][2g + rr]
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        const float2 l2 = lse2[4 * g];
        const uint64_t nl = f2_pack(-l2.x, -l2.y);
#pragma unroll
        for (int b = 0; b < 2; ++b) {
#pragma unroll
          for (int rr = 0; rr < 2; ++rr) {
            const uint64_t x =
                f2_fma(f2_pack(__uint_as_float(sr[b][4 * g + 2 * rr]), __uint_as_float(sr[b][4 * g + 2 * rr + 1])), c2, nl);
            if (((2 * g + rr) & 7) >= 8 - kEmuPairs) {
              pf[b][2 * g + rr] = ex2_fma2(x);
            } else {
              float x0, x1;
              f2_unpack(x, x0, x1);
              pf[b][2 * g + rr] = f2_pack(ex2(x0), ex2(x1));
            }
          }
        }
      }
      if (pad != 0 || diag) {  // padding key rows, or the tile is on the diagonal
#pragma unroll
        for (int b = 0; b < 2; ++b) {
#pragma unroll
          for (int rr = 0; rr < 2; ++rr) {
            const int k = 32 * wq + 16 * b + 8 * rr + g4;
            const bool dead = (pad >> (2 * b + rr)) & 1;
#pragma unroll
            for (int g = 0; g < 8; ++g) {
              const int q = 64 * h + 8 * g + 2 * t4;
              float p0, p1;
              f2_unpack(pf[b][2 * g + rr], p0, p1);
              if (dead || (diag && k > q)) p0 = 0.f;
              if (dead || (diag && k > q + 1)) p1 = 0.f;
              pf[b][2 * g + rr] = f2_pack(p0, p1);
            }
          }
        }
      }
      // 16-bit P^T over the first 32 columns of this half's scores: query pair
      // 2m, 2m+1 of the half in column m (m = 4g + t%4)
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          float p0, p1;
          f2_unpack(pf[b][e], p0, p1);
          pk[e] = E::pack2(p0, p1);
        }
        tmem_st16x128_x8(tS + (static_cast<uint32_t>(16 * b) << 16), pk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar_p);
      float2 dvv[8];  // this thread's D pairs, read while dP^T is being computed
#pragma unroll
      for (int g = 0; g < 8; ++g) dvv[g] = dv2[4 * g];

      if (!__all_sync(0xffffffffu, mbar_wait(bar_dp, g & 1, abort_flag, tmo, 221))) {
        ok = false;
        break;
      }
      if (g > 0 && !__all_sync(0xffffffffu, mbar_wait(bar_dsfree, (g - 1) & 1, abort_flag, tmo, 222))) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        uint32_t dpr[32];
        tmem_ld16x256_x8(tDP + (static_cast<uint32_t>(16 * b) << 16), dpr);
        tmem_wait_ld();
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          const uint64_t dd = f2_pack(dvv[g].x, dvv[g].y);
          uint32_t w[2];
#pragma unroll
          for (int rr = 0; rr < 2; ++rr) {
            const uint64_t ds2 = f2_mul(pf[b][2 * g + rr],
                                        f2_sub(f2_pack(__uint_as_float(dpr[4 * g + 2 * rr]),
                                                       __uint_as_float(dpr[4 * g + 2 * rr + 1])),
                                               dd));
            float d0, d1;
            f2_unpack(ds2, d0, d1);
            w[rr] = E::pack2(d0, d1);
          }
          // rows 32wq + 16b + (lane & 15): 8x8 matrices rr = 0, 1 of column group g
          stmatrix_x2(ds_lane + 16 * b * 128 + ((g ^ ds_sw) << 4), w[0], w[1]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar_ds);
    }
    if (!ok) break;
    // epilogue: half 0 writes dK (times scale), half 1 writes dV; the
    // accumulators are handed back once read
    if (!__all_sync(0xffffffffu, mbar_wait(bar_final, t & 1, abort_flag, tmo, 223))) {
      ok = false;
      break;
    }
    {
      tc_fence_after();
      int j, bh, i0, n_;
      unit_item(wu, half, j, bh, i0, n_);
      const int key = j * 128 + wq * 32 + lane;  // this thread's key row
      const bool key_ok = key < N;
      const uint32_t tAcc = tmem + lane_off + (h == 0 ? C::kColDK : C::kColDV);
      const float mul = (h == 0) ? p.scale : 1.0f;
      T* out = static_cast<T*>(h == 0 ? p.dk : p.dv) + (static_cast<size_t>(bh) * N + key) * D;
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t a[32];
        tmem_ld32(tAcc + 32 * cc, a);
        tmem_wait_ld();
        if (key_ok) {
          uint32_t w[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            w[e] = E::pack2(__uint_as_float(a[2 * e]) * mul, __uint_as_float(a[2 * e + 1]) * mul);
          uint4* dst = reinterpret_cast<uint4*>(out + 32 * cc);
#pragma unroll
          for (int e = 0; e < 4; ++e) dst[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
        }
      }
      tc_fence_before();
      mbar_arrive(bar_accfree);
    }
    g0_ += n;
    ++t_;
    }
  } else {
    setmaxnreg_inc<C::kRegsDrain>();
    // ------------------------------------------------------------ dQ drain
    // Warp w owns query rows [32 w, 32 w + 32) of the partial.  Columns go in
    // 64-wide passes through an 8 KB staging slice (at d = 128 in the dO
    // buffer of this step, which dV and dP have finished reading once the
    // partial is ready), laid out as two 32-column TMA boxes with 128-byte
    // swizzle; one lane then issues the TMA reduce-adds into the fp32
    // accumulator.  The slice is handed back (bar_doempty) once the TMA
    // engine has read it.
    const int wq = warp & 3;
    const uint32_t tQ = tmem + (static_cast<uint32_t>(wq * 32) << 16) + C::kColDQ;
    const uint32_t swz = static_cast<uint32_t>(lane & 7);
    bool ok = true;
    int g0_ = 0;
    for (int wu = blockIdx.x; wu < units && ok; wu += kPersist ? static_cast<int>(gridDim.x) : units)
    for (int half = 0; half < kHalves && ok; ++half) {
    int j, bh, i0, n;
    if (!unit_item(wu, half, j, bh, i0, n)) continue;
    const int g0 = kPersist ? g0_ : 0;  // this item's first step
    for (int it = 0; it < n; ++it) {
      const int g = g0 + it;
      const int st = g & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(bar_dqfull, g & 1, abort_flag, tmo, 230))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint8_t* stage = (D == 128 ? sDO + st * TILE : smem + C::kOffStage) + wq * 8192;
      uint8_t* my_row = stage + lane * 128;
      const int grow = bh * p.Np + (i0 + it) * 128 + wq * 32;  // first accumulator row of this warp
      uint32_t a[32], b[32], a2[32], b2[32];
      tmem_ld32(tQ, a);
      tmem_ld32(tQ + 32, b);
      if (D == 128) {
        tmem_ld32(tQ + 64, a2);
        tmem_ld32(tQ + 96, b2);
      }
      tmem_wait_ld();
      // every read of this partial is complete: hand the columns back
      tc_fence_before();
      mbar_arrive(bar_dqfree);
      // dV_i and dP_i have read dO_i: its buffer may take the staging, and
      // be handed back to the producer afterwards
      if (!__all_sync(0xffffffffu, mbar_wait(&bar_dvdone[st], (g >> 1) & 1, abort_flag, tmo, 232))) {
        ok = false;
        break;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        *reinterpret_cast<uint4*>(my_row + ((u ^ swz) << 4)) = make_uint4(a[4 * u], a[4 * u + 1], a[4 * u + 2], a[4 * u + 3]);
        *reinterpret_cast<uint4*>(my_row + 4096 + ((u ^ swz) << 4)) =
            make_uint4(b[4 * u], b[4 * u + 1], b[4 * u + 2], b[4 * u + 3]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_reduce_add_2d(stage, &p.tm_dq, 0, grow);
        tma_reduce_add_2d(stage + 4096, &p.tm_dq, 32, grow);
        bulk_commit_group();
      }
      if (D == 128) {
        if (lane == 0) bulk_wait_group_read0();  // the first pass has left shared memory
        __syncwarp();
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          *reinterpret_cast<uint4*>(my_row + ((u ^ swz) << 4)) =
              make_uint4(a2[4 * u], a2[4 * u + 1], a2[4 * u + 2], a2[4 * u + 3]);
          *reinterpret_cast<uint4*>(my_row + 4096 + ((u ^ swz) << 4)) =
              make_uint4(b2[4 * u], b2[4 * u + 1], b2[4 * u + 2], b2[4 * u + 3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_reduce_add_2d(stage, &p.tm_dq, 64, grow);
          tma_reduce_add_2d(stage + 4096, &p.tm_dq, 96, grow);
          bulk_commit_group();
        }
      }
      if (lane == 0) {
        bulk_wait_group_read0();
        mbar_arrive(&bar_doempty[st]);  // the producer may load the next dO into this stage
      }
      __syncwarp();
    }
    g0_ += n;
    }
    if (lane == 0) bulk_wait_group0();  // the additions have reached global memory
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------- stage 1
// One row per (d/8) lanes; each lane reads 8 elements (16 bytes) of O and dO.
template <int D, typename T>
__global__ void __launch_bounds__(256) attn_bwd_preprocess_kernel(const T* __restrict__ o, const T* __restrict__ dO,
                                                                  const float* __restrict__ lse,
                                                                  float* __restrict__ dvec,
                                                                  float* __restrict__ lse2,
                                                                  float* __restrict__ dq_acc, int BH, int N,
                                                                  int Np) {
  constexpr int LPR = D / 8;            // lanes per row
  constexpr int RPB = 256 / LPR;        // rows per block
  const int sub = threadIdx.x % LPR;
  const long long row = static_cast<long long>(blockIdx.x) * RPB + threadIdx.x / LPR;  // over BH * Np
  const long long total = static_cast<long long>(BH) * Np;
  float acc = 0.f;
  const bool in = row < total;
  const int bh = in ? static_cast<int>(row / Np) : 0;
  const int i = in ? static_cast<int>(row % Np) : 0;
  const bool valid = in && i < N;
  if (valid) {
    const size_t off = (static_cast<size_t>(bh) * N + i) * D + sub * 8;
    const uint4 a = *reinterpret_cast<const uint4*>(o + off);
    const uint4 b = *reinterpret_cast<const uint4*>(dO + off);
    const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 x = Elem<T>::unpack2(wa[e]);
      const float2 y = Elem<T>::unpack2(wb[e]);
      acc = fmaf(x.x, y.x, acc);
      acc = fmaf(x.y, y.y, acc);
    }
  }
#pragma unroll
  for (int m = LPR / 2; m > 0; m >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
  if (in) {
    float4* z = reinterpret_cast<float4*>(dq_acc + static_cast<size_t>(row) * D + sub * 8);
    z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (sub == 0) {
      dvec[row] = valid ? acc : 0.f;
      lse2[row] = valid ? lse[static_cast<size_t>(bh) * N + i] * 1.4426950408889634f : INFINITY;
    }
  }
}

template <typename T>
inline void launch_bwd_preprocess(const void* o, const void* dO, const float* lse, float* dvec, float* lse2,
                                  float* dq_acc, int BH, int N, int Np, int d, cudaStream_t s) {
  const long long rows = static_cast<long long>(BH) * Np;
  const T* ot = static_cast<const T*>(o);
  const T* dt = static_cast<const T*>(dO);
  if (d == 64) {
    const unsigned blocks = static_cast<unsigned>((rows + 31) / 32);
    attn_bwd_preprocess_kernel<64, T><<<blocks, 256, 0, s>>>(ot, dt, lse, dvec, lse2, dq_acc, BH, N, Np);
  } else {
    const unsigned blocks = static_cast<unsigned>((rows + 15) / 16);
    attn_bwd_preprocess_kernel<128, T><<<blocks, 256, 0, s>>>(ot, dt, lse, dvec, lse2, dq_acc, BH, N, Np);
  }
}

// ---------------------------------------------------------------- stage 3
// Each thread converts 8 consecutive elements of one row.
template <typename T>
__global__ void __launch_bounds__(256) attn_bwd_dq_convert_kernel(const float* __restrict__ dq_acc,
                                                                  T* __restrict__ dq, int N, int Np, int d,
                                                                  float scale, long long total8) {
  const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= total8) return;
  const long long e = t * 8;                    // element index in [BH, N, d]
  const long long rowN = e / d;                 // bh * N + i
  const int col = static_cast<int>(e - rowN * d);
  const long long bh = rowN / N;
  const long long i = rowN - bh * N;
  const float4* src = reinterpret_cast<const float4*>(dq_acc + (bh * Np + i) * d + col);
  const float4 a = src[0], b = src[1];
  uint4 w;
  w.x = Elem<T>::pack2(a.x * scale, a.y * scale);
  w.y = Elem<T>::pack2(a.z * scale, a.w * scale);
  w.z = Elem<T>::pack2(b.x * scale, b.y * scale);
  w.w = Elem<T>::pack2(b.z * scale, b.w * scale);
  *reinterpret_cast<uint4*>(dq + e) = w;
}

template <typename T>
inline void launch_bwd_dq_convert(const float* dq_acc, void* dq, int BH, int N, int Np, int d, float scale,
                                  cudaStream_t s) {
  const long long total8 = static_cast<long long>(BH) * N * d / 8;
  const unsigned blocks = static_cast<unsigned>((total8 + 255) / 256);
  attn_bwd_dq_convert_kernel<T><<<blocks, 256, 0, s>>>(dq_acc, static_cast<T*>(dq), N, Np, d, scale, total8);
}

}  // namespace exattn

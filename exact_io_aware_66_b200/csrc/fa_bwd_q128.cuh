// fa_bwd_q128.cuh — exact attention backward for sm_100a with 128-row query tiles (d = 64 and
// d = 128, and d = 96 through zero-filled columns; no dropout).
//
// Same mathematics as fa_bwd_main (fa_bwd.cuh): with P = exp(S - lse),
//     dV = P^T dO,  dP = dO V^T,  D_i = dO_i . O_i,  dS = P o (dP - D),
//     dQ = scale dS K,  dK = scale dS^T Q,
// recomputed on chip from Q, K, V, dO and the forward's logsumexp ("How FlashAttention Actually
// Works", section "The Backward Pass: Recomputation"), and the same preprocess and dQ
// conversion kernels around it. What differs is the tiling of the main kernel:
//
//   * a work unit is one (key/value head, 128-key tile j); the query tiles it visits are 128
//     rows, so every tcgen05 product is M = 128, N = 128 (an N = 64 product reads 6 KB of
//     shared-memory operands per k-step for half the work of an N = 128 one, which reads 8 KB).
//   * the kernel is persistent: one CTA per SM takes units from a grid-wide counter (zeroed by
//     the preprocess kernel) in the grouped longest-first order of grouped_unit, so one unit's
//     dK/dV epilogue and the next unit's start overlap, and no SM idles while another finishes
//     a long unit. Every pipeline barrier below counts its phases over the CTA's whole run.
//   * TMEM holds exactly four 128-column fp32 regions: dV, dK, S^T (then P^T in place) and dP^T
//     (then dQ^T in place; at d = 64, dQ = dS K with the queries on the lanes, since an M = 64
//     product would leave half the lanes idle). Nothing is double buffered; the MMA issue order is
//         S(i), dK(i-1), dQ(i-1), dP(i), dV(i), S(i+1), ...
//     so the elementwise warps turn S^T(i) into P^T(i) while the tensor core finishes tile i-1
//     and computes dP^T(i) (which does not wait for P^T(i)). At d = 64, where the products are
//     short, dP(i) and dV(i) go in whichever order their inputs arrive, so that dV(i) can fill
//     the wait for the drain of dQ(i-1) when P^T(i) is ready first.
//   * The drain warpgroup copies all of dQ^T(i) into registers and frees its TMEM columns at
//     once, then adds it into the fp32 accumulator with TMA bulk reductions
//     (cp.reduce.async.bulk .add.f32) from a 32 KB staging buffer. At the end of a unit it also
//     reads dV and dK out of TMEM (freeing them for the next unit's first products) and stores
//     them through the same staging buffer.
//   * Q tiles with their per-row terms (-lse log2e and D) travel in a 2-stage TMA ring; dO has a
//     single slot, refilled after dV(i), its last reader, and needed again by dP(i+1) three
//     products later. That single slot is what pays for the staging buffer. K and V of the
//     next unit load once the current unit's last product has completed.
//
// Shared memory at d = 128 (about 227 KB): K, V (32 KB each), two Q stages (64 KB), dO (32 KB),
// dS^T (32 KB), dQ staging (32 KB), two stages of per-row terms (2 KB), barriers; at d = 64 the
// five 128 x d tiles take half as much (163 KB in all). The 128-byte swizzle needs a 1024-byte
// aligned base; a misaligned base is reported through the status word (code 7) instead of
// being used.
#pragma once
#include "fa_bwd.cuh"

namespace fa {

template <int D>
struct Bwd128Layout {
  static constexpr int kBox = 128 * 64 * 2;        // TMA box: 128 rows x 64 bf16 columns (SW128)
  static constexpr int kBoxes = D / 64;            // boxes per 128-row tile
  static constexpr int kTile = kBoxes * kBox;      // 128 rows x D columns
  static constexpr int kK = 0;
  static constexpr int kV = kTile;
  static constexpr int kQ = 2 * kTile;             // + stage * kTile (2 stages)
  static constexpr int kDO = 4 * kTile;            // one slot
  static constexpr int kDS = 5 * kTile;            // dS^T [128 keys][128 queries], two 64-query boxes
  static constexpr int kDQ = kDS + 2 * kBox;       // drain staging, 32 KB (4 warps x 8 KB)
  static constexpr int kRow = kDQ + 2 * kBox;      // per Q stage (1 KB): lse2[128], then D[128]
  static constexpr int kBars = kRow + 2 * 1024;

  static constexpr int bKV = 0;                    // K and V of the unit
  static constexpr int bQFull = 1;                 // + stage: Q tile, lse2 and D
  static constexpr int bQEmpty = 3;                // + stage
  static constexpr int bOFull = 5;                 // dO tile
  static constexpr int bOEmpty = 6;
  static constexpr int bSFull = 7;                 // S^T(i) in TMEM
  static constexpr int bDPFull = 8;                // dP^T(i) in TMEM
  static constexpr int bPDone = 9;                 // P^T(i) in TMEM (256 arrivals)
  static constexpr int bDSDone = 10;               // dS^T(i) in shared memory (256 arrivals)
  static constexpr int bDQFull = 11;               // dQ^T(i) in TMEM; dS^T(i) and Q(i) read
  static constexpr int bDQFree = 12;               // dQ^T(i) copied out of TMEM (128 arrivals)
  static constexpr int bAccDone = 13;              // every product of the unit completed
  static constexpr int bAccFree = 14;              // dV, dK of the unit read out of TMEM (128)
  static constexpr int bDrain = 15;
  static constexpr int bSchedFull = 16;            // + slot: next unit index published
  static constexpr int bSchedEmpty = 18;           // + slot: read by every consuming warp
  static constexpr int kNumBars = 20;
  static constexpr int kSchedReaders = 13;         // warps 0-11 and the MMA thread

  static constexpr int kAbort = kBars + kNumBars * 8;
  static constexpr int kSched = kAbort + 8;        // two unit indices (-1: no unit left)
  static constexpr int kTmemSlot = kSched + 8;
  static constexpr int kBytes = kTmemSlot + 8;

  // TMEM columns
  static constexpr uint32_t tDV = 0, tDK = 128, tS = 256, tDP = 384;
};
static_assert(Bwd128Layout<128>::kBytes <= 227 * 1024, "q128 backward shared memory");
static_assert(Bwd128Layout<64>::kBytes <= 227 * 1024, "q128 backward shared memory");

// Register split (setmaxnreg, per warpgroup): the drain warpgroup holds its lanes' 128 dQ^T
// columns in registers while it stages them; the two elementwise warpgroups keep 64 fp32
// probabilities per thread between their two phases; the MMA/TMA warpgroup needs the least.
// The shares add up to the launch allocation.
struct Bwd128Regs {
  static constexpr uint32_t kLaunch = 128;  // registers per thread at launch (checked on the host)
  static constexpr uint32_t kElem = 128, kDrain = 160, kOther = 96;
  static_assert(128 * (2 * kElem + kDrain + kOther) == kBwdThreads * kLaunch,
                "q128 backward register split must equal the launch allocation");
};

template <uint32_t R>
__device__ __forceinline__ void bwd128_setmaxnreg() {
  static_assert(R % 8 == 0 && R >= 24 && R <= 256, "setmaxnreg range");
  if constexpr (R > Bwd128Regs::kLaunch)
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(R));
  else if constexpr (R < Bwd128Regs::kLaunch)
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(R));
}

// One work unit: key tile k0 of key/value head bh, visited by n_i = qgroup * n_qt query tiles
// (n_qt 128-row tiles from tile qi0, for each query head sharing the key/value head).
struct Bwd128Unit {
  int bh, k0, qi0, n_qt, n_i;
};

template <bool CAUSAL>
__device__ __forceinline__ Bwd128Unit bwd128_unit(int u, const BwdParams& p) {
  Bwd128Unit w;
  int j;
  grouped_unit(u, p.n_kv, p.BH_kv, p.group, j, w.bh);
  w.k0 = 128 * j;
  // first 128-row query tile with a query that sees a key of this tile (j <= i + off)
  w.qi0 = CAUSAL ? max(0, w.k0 - p.off) / 128 : 0;
  w.n_qt = max(0, p.n_q - w.qi0);
  w.n_i = p.qgroup * w.n_qt;
  return w;
}

// D: the shared-memory and TMEM layout (64 or 128 columns of d). DM: the head dimension the
// products run over (D, or 96 with the d = 128 layout; the tensor maps zero-fill columns past d,
// so a 96-column contraction over them is exact).
template <int D, bool CAUSAL, int DM = D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    fa_bwd_main_q128(const __grid_constant__ CUtensorMap tmQ,
                     const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV,
                     const __grid_constant__ CUtensorMap tmDO,
                     const __grid_constant__ CUtensorMap tmLse2,
                     const __grid_constant__ CUtensorMap tmD,
                     const __grid_constant__ CUtensorMap tmDQacc,
                     const __grid_constant__ CUtensorMap tmDK,
                     const __grid_constant__ CUtensorMap tmDV, const BwdParams p) {
  using L = Bwd128Layout<D>;
  using R = Bwd128Regs;
  // No static shared memory in this kernel, so the dynamic block starts at the beginning of
  // the CTA's shared window. The layout uses all of it (no slack to realign), so the 1024-byte
  // alignment the swizzled operands need is checked rather than assumed. (An alignment
  // attribute on this declaration would raise the dynamic-block alignment of every kernel in
  // the library and push those with static shared memory over the limit.)
  extern __shared__ uint8_t smem_raw[];
  const uint32_t sbase = smem_u32(smem_raw);
  if (sbase & 1023u) {
    if (threadIdx.x == 0) atomicExch(p.status, 7);
    return;
  }
  uint8_t* gbase = smem_raw;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + L::kAbort);
  volatile int* sched = reinterpret_cast<volatile int*>(gbase + L::kSched);
  auto bar = [&](int i) -> uint32_t { return sbase + L::kBars + 8u * i; };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(bar(L::bKV), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(L::bQFull + s), 1);
      mbar_init(bar(L::bQEmpty + s), 1);
      mbar_init(bar(L::bSchedFull + s), 1);
      mbar_init(bar(L::bSchedEmpty + s), L::kSchedReaders);
    }
    mbar_init(bar(L::bOFull), 1);
    mbar_init(bar(L::bOEmpty), 1);
    mbar_init(bar(L::bSFull), 1);
    mbar_init(bar(L::bDPFull), 1);
    mbar_init(bar(L::bPDone), 256);
    mbar_init(bar(L::bDSDone), 256);
    mbar_init(bar(L::bDQFull), 1);
    mbar_init(bar(L::bDQFree), 128);
    mbar_init(bar(L::bAccDone), 1);
    mbar_init(bar(L::bAccFree), 128);
    mbar_init(bar(L::bDrain), 1);
    fence_barrier_init();
  }
  if (warp == 12) {
    tmem_alloc(sbase + L::kTmemSlot, 512);
    tmem_relinquish();
  }
  if (warp == 13 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmDO);
    tma_prefetch_desc(&tmDQacc);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(gbase + L::kTmemSlot);

  // Unit number s of this CTA, as a whole warp: wait for the TMA thread to publish it, then
  // acknowledge the read (one arrival per warp). -1: no unit left; kGaveUp: the wait gave up.
  constexpr int kGaveUp = -2;
  auto warp_next_unit = [&](int s) -> int {
    if (!warp_wait(bar(L::bSchedFull + (s & 1)), (s >> 1) & 1, abort_flag)) return kGaveUp;
    const int u = sched[s & 1];
    __syncwarp();
    if (lane == 0) mbar_arrive(bar(L::bSchedEmpty + (s & 1)));
    return u;
  };

  if (warp < 8) {
    // --------------------------------------------------- P^T and dS^T (elementwise) -----
    bwd128_setmaxnreg<R::kElem>();
    const int w = warp >> 2;                       // query columns [64w, 64w+64) of the tile
    const int r = threadIdx.x & 127;               // key row within the tile (TMEM lane)
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint64_t sl2x2 = f2_pack(p.scale_log2, p.scale_log2);
    uint8_t* dsb = gbase + L::kDS + w * L::kBox;
    bool ok = true;
    int g = 0;  // tiles of this CTA's earlier units
    for (int s = 0; ok; ++s) {
      const int u = warp_next_unit(s);
      if (u == kGaveUp) { ok = false; break; }
      if (u < 0) break;
      const Bwd128Unit U = bwd128_unit<CAUSAL>(u, p);
      const int key = U.k0 + r;
      for (int i = 0; i < U.n_i; ++i, ++g) {
        const int st = g & 1;
        const uint32_t ph = (g >> 1) & 1;
        const int qbase = 128 * (U.qi0 + i % U.n_qt) + 64 * w;
        const bool need_mask = (CAUSAL && qbase + p.off < U.k0 + 127) || (qbase + 64 > p.N) ||
                               (U.k0 + 128 > p.N_kv);
        // Phase 1: P = 2^(S scale log2e - lse log2e), kept in registers (fp32) and written to
        // TMEM as bf16 pairs over the first half of this warpgroup's S^T columns.
        ok = warp_wait(bar(L::bQFull + st), ph, abort_flag) &&
             warp_wait(bar(L::bSFull), g & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        const float* lse2 = reinterpret_cast<const float*>(gbase + L::kRow + st * 1024) + 64 * w;
        float pr[64];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t sv[32];
          tmem_ld_32x32b_x32(tmem + L::tS + 64 * w + 32 * h + lane_off, sv);
          tmem_ld_wait();
          reg_fence(sv);
#pragma unroll
          for (int c = 0; c < 32; c += 4) {
            const float4 l4 = *reinterpret_cast<const float4*>(lse2 + 32 * h + c);
            float a[4];
            f2_unpack(f2_fma(f2_pack_u(sv[c], sv[c + 1]), sl2x2, f2_pack(l4.x, l4.y)), a[0], a[1]);
            f2_unpack(f2_fma(f2_pack_u(sv[c + 2], sv[c + 3]), sl2x2, f2_pack(l4.z, l4.w)), a[2],
                      a[3]);
#pragma unroll
            for (int e = 0; e < 4; ++e) pr[32 * h + c + e] = ex2_approx(a[e]);
          }
          if (need_mask) {
            // valid queries of this chunk: lo <= c < hi (causal lower bound, sequence end), and
            // the key itself inside the sequence
            const int q0c = qbase + 32 * h;
            int lo = CAUSAL ? key - p.off - q0c : 0;
            int hi = p.N - q0c;
            if (key >= p.N_kv) lo = 32;
#pragma unroll
            for (int c = 0; c < 32; ++c)
              if (c < lo || c >= hi) pr[32 * h + c] = 0.f;
          }
          uint32_t pk[16];
#pragma unroll
          for (int c = 0; c < 16; ++c)
            pk[c] = pack_bf16x2(pr[32 * h + 2 * c], pr[32 * h + 2 * c + 1]);
          tmem_st_32x32b_x16(tmem + L::tS + 64 * w + 16 * h + lane_off, pk);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(bar(L::bPDone));
        // Phase 2: dS = P o (dP - D) to shared memory (bf16, MN-major for dQ's operand) and to
        // TMEM (dK's A operand), once dQ of the previous tile has read the previous dS.
        ok = warp_wait(bar(L::bDPFull), g & 1, abort_flag) &&
             (g == 0 || warp_wait(bar(L::bDQFull), (g - 1) & 1, abort_flag));
        if (!ok) break;
        tc_fence_after();
        const float* Dv =
            reinterpret_cast<const float*>(gbase + L::kRow + st * 1024 + 512) + 64 * w;
#pragma unroll
        for (int h = 0; h < 4; ++h) {  // 16 queries at a time
          uint32_t dp[16];
          tmem_ld_32x32b_x16(tmem + L::tDP + 64 * w + 16 * h + lane_off, dp);
          tmem_ld_wait();
          reg_fence(dp);
          uint32_t dsk[8];
#pragma unroll
          for (int c = 0; c < 16; c += 4) {
            const float4 d4 = *reinterpret_cast<const float4*>(Dv + 16 * h + c);
            float dsr[4];
            f2_unpack(f2_mul(f2_pack(pr[16 * h + c], pr[16 * h + c + 1]),
                             f2_sub(f2_pack_u(dp[c], dp[c + 1]), f2_pack(d4.x, d4.y))),
                      dsr[0], dsr[1]);
            f2_unpack(f2_mul(f2_pack(pr[16 * h + c + 2], pr[16 * h + c + 3]),
                             f2_sub(f2_pack_u(dp[c + 2], dp[c + 3]), f2_pack(d4.z, d4.w))),
                      dsr[2], dsr[3]);
            dsk[c / 2] = pack_bf16x2(dsr[0], dsr[1]);
            dsk[c / 2 + 1] = pack_bf16x2(dsr[2], dsr[3]);
          }
#pragma unroll
          for (int t = 0; t < 2; ++t)
            *reinterpret_cast<uint4*>(dsb + sw128_offset(r, 2 * h + t)) =
                make_uint4(dsk[4 * t], dsk[4 * t + 1], dsk[4 * t + 2], dsk[4 * t + 3]);
          // and to TMEM over this warpgroup's first dP^T columns, already read (piece h writes
          // columns 64w + 8h .. 64w + 8h + 7, below the ones it read): the A operand of dK
          tmem_st_32x32b_x8(tmem + L::tDP + 64 * w + 8 * h + lane_off, dsk);
        }
        tmem_st_wait();
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(bar(L::bDSDone));
      }
    }
    if (!ok) fail(p.status, abort_flag, 5);
  } else if (warp < 12) {
    // ------------------------------------------ dQ drain, and the unit's dK / dV -----------
    bwd128_setmaxnreg<R::kDrain>();
    const int wq = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const float scale = p.scale;
    float* stagef = reinterpret_cast<float*>(gbase + L::kDQ + wq * 8192);
    uint8_t* stageb = gbase + L::kDQ + wq * 8192;
    const uint32_t stage_s = sbase + L::kDQ + wq * 8192;
    bool ok = true;
    int g = 0, uc = 0;  // tiles of earlier units; earlier units with at least one tile
    for (int s = 0; ok; ++s) {
      const int u = warp_next_unit(s);
      if (u == kGaveUp) { ok = false; break; }
      if (u < 0) break;
      const Bwd128Unit U = bwd128_unit<CAUSAL>(u, p);
      for (int i = 0; i < U.n_i; ++i, ++g) {
        if (!warp_wait(bar(L::bDQFull), g & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const int q0 = 128 * (U.qi0 + i % U.n_qt), qh = U.bh * p.qgroup + i / U.n_qt;
        if constexpr (D == 64) {
          // dQ(i) sits in TMEM as [128 queries (lanes)][64 columns]: warp wq holds queries
          // [32 wq, 32 wq + 32) and stages them as two 32 x 32 fp32 boxes in the 128-byte
          // swizzled layout (16-byte stores, conflict-free), each added into the accumulator by
          // one TMA reduction.
          uint32_t v[64];
#pragma unroll
          for (int c = 0; c < 2; ++c)
            tmem_ld_32x32b_x32(tmem + L::tDP + 32 * c + lane_off,
                               *reinterpret_cast<uint32_t(*)[32]>(&v[32 * c]));
          tmem_ld_wait();
          reg_fence(v);
          tc_fence_before();
          mbar_arrive(bar(L::bDQFree));
          const int qw = q0 + 32 * wq;
          if (qw >= p.N) continue;  // no rows of this warp's slice exist
          if (lane == 0) bulk_wait_group_read0();  // the previous bulk copy has read the staging
          __syncwarp();
#pragma unroll
          for (int b = 0; b < 2; ++b)
#pragma unroll
            for (int t = 0; t < 8; ++t)
              *reinterpret_cast<float4*>(stageb + b * 4096 + sw128_offset(lane, t)) =
                  make_float4(__uint_as_float(v[32 * b + 4 * t]) * scale,
                              __uint_as_float(v[32 * b + 4 * t + 1]) * scale,
                              __uint_as_float(v[32 * b + 4 * t + 2]) * scale,
                              __uint_as_float(v[32 * b + 4 * t + 3]) * scale);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_reduce_add_3d(&tmDQacc, stage_s, 0, qw, qh);
            tma_reduce_add_3d(&tmDQacc, stage_s + 4096, 32, qw, qh);
            bulk_commit_group();
          }
        } else {
          // dQ^T(i) sits in TMEM as [d (lanes)][128 queries]: warp wq holds rows
          // [32 wq, 32 wq + 32) of d (rows past d = 96 are zero and skipped). All of it comes
          // into registers first, so the MMA can reuse the columns at once.
          uint32_t v[128];
#pragma unroll
          for (int c = 0; c < 4; ++c)
            tmem_ld_32x32b_x32(tmem + L::tDP + 32 * c + lane_off,
                               *reinterpret_cast<uint32_t(*)[32]>(&v[32 * c]));
          tmem_ld_wait();
          reg_fence(v);
          tc_fence_before();
          mbar_arrive(bar(L::bDQFree));
          if (32 * wq >= p.d) continue;
#pragma unroll
          for (int hq = 0; hq < 2; ++hq) {
            if (q0 + 64 * hq >= p.N) break;  // no rows of this half exist
            if (lane == 0) bulk_wait_group_read0();
            __syncwarp();
            // staging box: 64 query rows x 32 columns (this warp's d slice), fp32
#pragma unroll
            for (int q = 0; q < 64; ++q)
              stagef[q * 32 + lane] = __uint_as_float(v[64 * hq + q]) * scale;
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_reduce_add_3d(&tmDQacc, stage_s, 32 * wq, q0 + 64 * hq, qh);
              bulk_commit_group();
            }
          }
        }
      }
      if (!ok) break;
      // dV and dK * scale of the unit (zero when no query sees its keys): TMEM -> bf16 ->
      // staging (32 rows x 64 columns per 4 KB box, 128-byte swizzle) -> TMA store. dK goes to
      // registers right after dV, so TMEM is released before the stores.
      const bool has = U.n_i > 0;
      if (has) {
        if (!warp_wait(bar(L::bAccDone), uc & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
      }
      const int row0 = U.k0 + 32 * wq;
      if (lane == 0) bulk_wait_group_read0();
      __syncwarp();
#pragma unroll
      for (int c = 0; c < DM; c += 32) {
        uint32_t v[32];
        if (has) {
          tmem_ld_32x32b_x32(tmem + L::tDV + c + lane_off, v);
          tmem_ld_wait();
          reg_fence(v);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = 0u;
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int chunk = c / 8 + q;
          *reinterpret_cast<uint4*>(stageb + (chunk >> 3) * 4096 + sw128_offset(lane, chunk & 7)) =
              make_uint4(pack_bf16x2(__uint_as_float(v[8 * q]), __uint_as_float(v[8 * q + 1])),
                         pack_bf16x2(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3])),
                         pack_bf16x2(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5])),
                         pack_bf16x2(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7])));
        }
      }
      uint32_t dk[DM / 2];
#pragma unroll
      for (int c = 0; c < DM; c += 32) {
        uint32_t v[32];
        if (has) {
          tmem_ld_32x32b_x32(tmem + L::tDK + c + lane_off, v);
          tmem_ld_wait();
          reg_fence(v);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = 0u;
        }
#pragma unroll
        for (int e = 0; e < 16; ++e)
          dk[c / 2 + e] = pack_bf16x2(__uint_as_float(v[2 * e]) * scale,
                                      __uint_as_float(v[2 * e + 1]) * scale);
      }
      if (has) {
        tc_fence_before();
        mbar_arrive(bar(L::bAccFree));
        ++uc;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
#pragma unroll
        for (int bx = 0; bx < L::kBoxes; ++bx)
          tma_store_3d(&tmDV, stage_s + bx * 4096, 64 * bx, row0, U.bh);
        bulk_commit_group();
      }
      // at d = 64 dV and dK sit side by side in the 8 KB; at d = 128 dK reuses dV's space
      constexpr int kDKOff = D == 64 ? 4096 : 0;
      if constexpr (D == 128) {
        if (lane == 0) bulk_wait_group_read0();
        __syncwarp();
      }
#pragma unroll
      for (int chunk = 0; chunk < DM / 8; ++chunk)
        *reinterpret_cast<uint4*>(stageb + kDKOff + (chunk >> 3) * 4096 +
                                  sw128_offset(lane, chunk & 7)) =
            make_uint4(dk[4 * chunk], dk[4 * chunk + 1], dk[4 * chunk + 2], dk[4 * chunk + 3]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
#pragma unroll
        for (int bx = 0; bx < L::kBoxes; ++bx)
          tma_store_3d(&tmDK, stage_s + kDKOff + bx * 4096, 64 * bx, row0, U.bh);
        bulk_commit_group();
      }
    }
    if (!ok) fail(p.status, abort_flag, 5);
    if (lane == 0) bulk_wait_group0();
  } else {
    bwd128_setmaxnreg<R::kOther>();
    if (warp == 12 && lane == 0) {
      // ------------------------------------------------------------------- MMA ----------
      const uint32_t id_s = idesc_bf16_f32(128, 128, false, false);  // S^T, dP^T
      const uint32_t id_acc = idesc_bf16_f32(128, DM, false, true);  // dV, dK
      const uint32_t id_dq = idesc_bf16_f32(128, D, true, true);     // dQ^T (d = 128), dQ (64)
      const uint64_t dK_k = sdesc_sw128(sbase + L::kK, 16, 1024);          // K, K-major
      const uint64_t dV_k = sdesc_sw128(sbase + L::kV, 16, 1024);          // V, K-major
      const uint64_t dKt_mn = sdesc_sw128(sbase + L::kK, L::kBox, 1024);   // K^T, MN-major
      const uint64_t dQ_k = sdesc_sw128(sbase + L::kQ, 16, 1024);          // Q, K-major
      const uint64_t dDO_k = sdesc_sw128(sbase + L::kDO, 16, 1024);        // dO, K-major
      const uint64_t dQ_mn = sdesc_sw128(sbase + L::kQ, L::kBox, 1024);    // Q, MN-major
      const uint64_t dDO_mn = sdesc_sw128(sbase + L::kDO, L::kBox, 1024);  // dO, MN-major
      const uint64_t dDS_mn = sdesc_sw128(sbase + L::kDS, L::kBox, 1024);  // dS^T, MN-major
      // K-step kk of a K-major operand: box kk / 4, 32 bytes per step inside the 128-byte row;
      // of an MN-major operand: 16 rows of 128 bytes.
      auto kmaj = [](int kk) { return static_cast<uint32_t>((kk >> 2) * L::kBox + (kk & 3) * 32); };
      auto mma_s = [&](int st) {  // S^T = K Q^T, Q from stage st
        const uint32_t so = static_cast<uint32_t>(st) * L::kTile;
#pragma unroll
        for (int kk = 0; kk < DM / 16; ++kk)
          umma_ss(tmem + L::tS, sdesc_advance(dK_k, kmaj(kk)), sdesc_advance(dQ_k, so + kmaj(kk)),
                  id_s, kk > 0 ? 1u : 0u);
      };
      auto mma_dp = [&]() {  // dP^T = V dO^T
#pragma unroll
        for (int kk = 0; kk < DM / 16; ++kk)
          umma_ss(tmem + L::tDP, sdesc_advance(dV_k, kmaj(kk)), sdesc_advance(dDO_k, kmaj(kk)),
                  id_s, kk > 0 ? 1u : 0u);
      };
      auto mma_dv = [&](bool acc) {  // dV += P^T dO; P^T from TMEM (warpgroup w's queries at 64w)
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_ts(tmem + L::tDV, tmem + L::tS + (kk >> 2) * 64 + (kk & 3) * 8,
                  sdesc_advance(dDO_mn, kk * 2048), id_acc, (kk > 0 || acc) ? 1u : 0u);
      };
      auto mma_dk = [&](int st, bool acc) {  // dK += dS^T Q; dS^T from TMEM (over dP^T)
        const uint32_t so = static_cast<uint32_t>(st) * L::kTile;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_ts(tmem + L::tDK, tmem + L::tDP + (kk >> 2) * 64 + (kk & 3) * 8,
                  sdesc_advance(dQ_mn, so + kk * 2048), id_acc, (kk > 0 || acc) ? 1u : 0u);
      };
      auto mma_dq = [&]() {  // into the dP^T columns
        if constexpr (D == 128) {  // dQ^T = K^T dS^T: M = d
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_ss(tmem + L::tDP, sdesc_advance(dKt_mn, kk * 2048),
                    sdesc_advance(dDS_mn, kk * 2048), id_dq, kk > 0 ? 1u : 0u);
        } else {  // dQ = dS K: M = 128 queries (dS^T read MN-major), N = d = 64 (K, MN-major)
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_ss(tmem + L::tDP, sdesc_advance(dDS_mn, kk * 2048),
                    sdesc_advance(dKt_mn, kk * 2048), id_dq, kk > 0 ? 1u : 0u);
        }
      };
      const uint64_t lim = p.limit_ns;
      bool ok = true;
      int g = 0, uc = 0;  // tiles of earlier units; earlier units with at least one tile
      for (int s = 0; ok; ++s) {
        if (!(ok = mbar_wait(bar(L::bSchedFull + (s & 1)), (s >> 1) & 1, abort_flag, lim))) break;
        const int u = sched[s & 1];
        mbar_arrive(bar(L::bSchedEmpty + (s & 1)));
        if (u < 0) break;
        const int n_i = bwd128_unit<CAUSAL>(u, p).n_i;
        if (n_i == 0) continue;
        if (!(ok = mbar_wait(bar(L::bKV), uc & 1, abort_flag, lim))) break;
        for (int i = 0; i <= n_i && ok; ++i) {
          const int gi = g + i;
          if (i < n_i) {
            if (!(ok = mbar_wait(bar(L::bQFull + (gi & 1)), (gi >> 1) & 1, abort_flag, lim))) break;
            tc_fence_after();
            mma_s(gi & 1);
            umma_commit(bar(L::bSFull));
          }
          if (i > 0) {
            if (!(ok = mbar_wait(bar(L::bDSDone), (gi - 1) & 1, abort_flag, lim))) break;
            tc_fence_after();
            mma_dk((gi - 1) & 1, i > 1);
            umma_commit(bar(L::bQEmpty + ((gi - 1) & 1)));
            mma_dq();
            umma_commit(bar(L::bDQFull));
          }
          // dP(i) needs dO(i) and its TMEM columns back from the drain; dV(i) needs dO(i) and
          // P^T(i), and the unit's first dV also the previous unit's dV, dK read out of TMEM.
          // Neither waits for the other.
          const bool need_acc = i == 0 && uc > 0;
          if (i < n_i && D == 64) {
            // short products: whichever is ready first goes first (dV(i) then covers the drain
            // of dQ(i-1) when P^T(i) is ready before it)
            bool dp_done = false, dv_done = false;
            const uint64_t t0 = globaltimer_ns();
            for (uint32_t it = 0; !(dp_done && dv_done); ++it) {
              if (!dp_done && mbar_test(bar(L::bOFull), gi & 1) &&
                  (gi == 0 || mbar_test(bar(L::bDQFree), (gi - 1) & 1))) {
                tc_fence_after();
                mma_dp();
                umma_commit(bar(L::bDPFull));
                dp_done = true;
              }
              if (!dv_done && mbar_test(bar(L::bOFull), gi & 1) &&
                  mbar_test(bar(L::bPDone), gi & 1) &&
                  (!need_acc || mbar_test(bar(L::bAccFree), (uc - 1) & 1))) {
                tc_fence_after();
                mma_dv(i > 0);
                dv_done = true;
              }
              if (!(dp_done && dv_done)) {
                __nanosleep(32);
                if ((it & 63u) == 63u && (*abort_flag || globaltimer_ns() - t0 > lim)) {
                  ok = false;
                  break;
                }
              }
            }
            if (!ok) break;
            umma_commit(bar(L::bOEmpty));  // dO(i)'s readers, dP(i) and dV(i), have completed
          } else if (i < n_i) {
            // long products: dP(i) first, so that the elementwise warps find it complete when
            // they finish P^T(i)
            if (!(ok = mbar_wait(bar(L::bOFull), gi & 1, abort_flag, lim))) break;
            if (gi > 0 && !(ok = mbar_wait(bar(L::bDQFree), (gi - 1) & 1, abort_flag, lim)))
              break;
            tc_fence_after();
            mma_dp();
            umma_commit(bar(L::bDPFull));
            if (!(ok = mbar_wait(bar(L::bPDone), gi & 1, abort_flag, lim))) break;
            if (need_acc && !(ok = mbar_wait(bar(L::bAccFree), (uc - 1) & 1, abort_flag, lim)))
              break;
            tc_fence_after();
            mma_dv(i > 0);
            umma_commit(bar(L::bOEmpty));  // dV(i) is dO(i)'s last reader
          }
        }
        if (!ok) break;
        umma_commit(bar(L::bAccDone));
        g += n_i;
        ++uc;
      }
      if (!ok) fail(p.status, abort_flag, 5);
      // Every MMA this thread issued completes before tensor memory is freed (the drain after a
      // give-up; on the normal path the epilogue waits for the same products). Bounded wait.
      volatile int never = 0;
      umma_commit(bar(L::bDrain));
      mbar_wait(bar(L::bDrain), 0, &never);
    } else if (warp == 13 && lane == 0) {
      // ------------------------------------------------- TMA, and the unit scheduler ----------
      bool ok = true;
      int g = 0, uc = 0;
      int issued_o = 0, issued_q = 0, skipped = -1, kv_loads = 0;
      int u = static_cast<int>(blockIdx.x);
      for (int s = 0;; ++s) {
        // publish unit s of this CTA (-1 when none is left) once every reader has taken unit s-2
        if (!mbar_wait(bar(L::bSchedEmpty + (s & 1)), ((s >> 1) & 1) ^ 1, abort_flag)) {
          ok = false;
          break;
        }
        const int pub = u < p.n_units ? u : -1;
        sched[s & 1] = pub;
        mbar_arrive(bar(L::bSchedFull + (s & 1)));
        if (pub < 0) break;
        const Bwd128Unit U = bwd128_unit<CAUSAL>(u, p);
        for (int i = 0; i < U.n_i; ++i) {
          const int gi = g + i, st = gi & 1;
          const int q0 = 128 * (U.qi0 + i % U.n_qt), qh = U.bh * p.qgroup + i / U.n_qt;
          const uint32_t so = static_cast<uint32_t>(st) * L::kTile;
          // Q(i) with its row terms: the stage frees after dK of the tile two back
          if (!mbar_wait(bar(L::bQEmpty + st), ((gi >> 1) & 1) ^ 1, abort_flag)) {
            ok = false;
            break;
          }
          if (i != p.dbg_skip) {  // (the test hook leaves this tile out)
            mbar_arrive_expect_tx(bar(L::bQFull + st), L::kTile + 1024);
#pragma unroll
            for (int bx = 0; bx < L::kBoxes; ++bx)
              tma_load_3d(sbase + L::kQ + so + bx * L::kBox, &tmQ, bar(L::bQFull + st), 64 * bx,
                          q0, qh);
            tma_load_3d(sbase + L::kRow + st * 1024, &tmLse2, bar(L::bQFull + st), q0, qh, 0);
            tma_load_3d(sbase + L::kRow + st * 1024 + 512, &tmD, bar(L::bQFull + st), q0, qh, 0);
          } else {
            skipped = gi;
          }
          issued_q = gi + 1;
          // dO(i): the single slot frees after dV of the previous tile
          if (gi > 0 && !mbar_wait(bar(L::bOEmpty), (gi - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar(L::bOFull), L::kTile);
#pragma unroll
          for (int bx = 0; bx < L::kBoxes; ++bx)
            tma_load_3d(sbase + L::kDO + bx * L::kBox, &tmDO, bar(L::bOFull), 64 * bx, q0, qh);
          issued_o = gi + 1;
          if (i == 0) {
            // K and V of the unit, once every product of the previous unit has completed
            if (uc > 0 && !mbar_wait(bar(L::bAccDone), (uc - 1) & 1, abort_flag)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(bar(L::bKV), 2 * L::kTile);
#pragma unroll
            for (int bx = 0; bx < L::kBoxes; ++bx) {
              tma_load_3d(sbase + L::kK + bx * L::kBox, &tmK, bar(L::bKV), 64 * bx, U.k0, U.bh);
              tma_load_3d(sbase + L::kV + bx * L::kBox, &tmV, bar(L::bKV), 64 * bx, U.k0, U.bh);
            }
            kv_loads = uc + 1;
          }
        }
        if (!ok) break;
        if (U.n_i > 0) {
          g += U.n_i;
          ++uc;
        }
        u = static_cast<int>(gridDim.x) + atomicAdd(p.sched_counter, 1);
      }
      if (!ok) fail(p.status, abort_flag, 5);
      // Every load issued lands before the CTA can exit, whether or not (or whenever) a role
      // gives up; these are the latest loads of their slots, so on the normal path the bounded
      // waits return at once.
      volatile int never = 0;
      if (issued_o > 0) mbar_wait(bar(L::bOFull), (issued_o - 1) & 1, &never);
      for (int i = max(0, issued_q - 2); i < issued_q; ++i)
        if (i != skipped) mbar_wait(bar(L::bQFull + (i & 1)), (i >> 1) & 1, &never);
      if (kv_loads > 0) mbar_wait(bar(L::bKV), (kv_loads - 1) & 1, &never);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 12) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace fa

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
//   * one CTA per (key/value head, 128-key tile j); the query tiles it visits are 128 rows, so
//     every tcgen05 product is M = 128, N = 128 (an N = 64 product reads 6 KB of shared-memory
//     operands per k-step for half the work of an N = 128 one, which reads 8 KB).
//   * TMEM holds exactly four 128-column fp32 regions: dV, dK, S^T (then P^T in place) and dP^T
//     (then dQ^T in place; at d = 64, dQ = dS K with the queries on the lanes, since an M = 64
//     product would leave half the lanes idle). Nothing is double buffered; the MMA issue order is
//         S(i), dK(i-1), dQ(i-1), dV(i), dP(i), S(i+1), ...
//     so the elementwise warps turn S^T(i) into P^T(i) while the tensor core finishes tile i-1,
//     and the dQ^T(i-1) drain overlaps dV(i).
//   * The drain copies all of dQ^T(i) into registers and frees its TMEM columns at once, then
//     adds it into the fp32 accumulator with TMA bulk reductions (cp.reduce.async.bulk .add.f32)
//     from a 32 KB staging buffer, two 64-query halves per tile.
//   * Q tiles with their per-row terms (-lse log2e and D) travel in a 2-stage TMA ring; dO has a
//     single slot, refilled after dP(i), its last reader, and needed again by dV(i+1) three
//     products later. That single slot is what pays for the staging buffer.
//
// Shared memory at d = 128 (about 227 KB): K, V (32 KB each), two Q stages (64 KB), dO (32 KB),
// dS^T (32 KB), dQ staging (32 KB), two stages of per-row terms (2 KB), barriers; at d = 64 the
// five 128 x d tiles take half as much (163 KB in all). The 128-byte
// swizzle needs a 1024-byte aligned base; a misaligned base is reported through the status word
// (code 7) instead of being used.
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
  static constexpr int kDQ = kDS + 2 * kBox;       // dQ staging, 32 KB (4 warps x 8 KB)
  static constexpr int kRow = kDQ + 2 * kBox;      // per Q stage (1 KB): lse2[128], then D[128]
  static constexpr int kBars = kRow + 2 * 1024;

  static constexpr int bKV = 0;
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
  static constexpr int bAccDone = 13;
  static constexpr int bDrain = 14;
  static constexpr int kNumBars = 15;

  static constexpr int kAbort = kBars + kNumBars * 8;
  static constexpr int kTmemSlot = kAbort + 8;
  static constexpr int kBytes = kTmemSlot + 8;

  // TMEM columns
  static constexpr uint32_t tDV = 0, tDK = 128, tS = 256, tDP = 384;
};
static_assert(Bwd128Layout<128>::kBytes <= 227 * 1024, "q128 backward shared memory");
static_assert(Bwd128Layout<64>::kBytes <= 227 * 1024, "q128 backward shared memory");

// Register split (setmaxnreg, per warpgroup): the drain warpgroup holds its lanes' 128 dQ^T
// columns in registers while it stages them; the two elementwise warpgroups (64 fp32
// probabilities per thread between their two phases) and the MMA/TMA warpgroup give up the
// difference. The shares add up to the launch allocation.
struct Bwd128Regs {
  static constexpr uint32_t kLaunch = 128;  // registers per thread at launch (checked on the host)
  static constexpr uint32_t kElem = 120, kDrain = 168, kOther = 104;
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

template <int D, bool CAUSAL>
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
  auto bar = [&](int i) -> uint32_t { return sbase + L::kBars + 8u * i; };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Scheduling as in fa_bwd_main: groups of p.group key/value heads sized for L2; inside a
  // group the key tiles with the most query tiles first (longest-processing-time order).
  int j, bh;  // key tile, key/value head
  grouped_unit(static_cast<int>(blockIdx.x), p.n_kv, p.BH_kv, p.group, j, bh);
  const int k0 = 128 * j;
  // First 128-row query tile with a query that sees a key of this tile (j <= i + off); the
  // iterations run over every query head sharing this key/value head, times its query tiles.
  const int qi0 = CAUSAL ? max(0, k0 - p.off) / 128 : 0;
  const int n_qt = max(0, p.n_q - qi0);
  const int n_i = p.qgroup * n_qt;
  auto q_head = [&](int it) { return bh * p.qgroup + it / n_qt; };
  auto q_tile = [&](int it) { return qi0 + it % n_qt; };

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(bar(L::bKV), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(L::bQFull + s), 1);
      mbar_init(bar(L::bQEmpty + s), 1);
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

  if (warp < 8) {
    // --------------------------------------------------- P^T and dS^T (elementwise) -----
    bwd128_setmaxnreg<R::kElem>();
    const int w = warp >> 2;                       // query columns [64w, 64w+64) of the tile
    const int r = threadIdx.x & 127;               // key row within the tile (TMEM lane)
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int key = k0 + r;
    const uint64_t sl2x2 = f2_pack(p.scale_log2, p.scale_log2);
    uint8_t* dsb = gbase + L::kDS + w * L::kBox;
    bool ok = true;
    for (int i = 0; i < n_i && ok; ++i) {
      const int st = i & 1;
      const uint32_t ph = (i >> 1) & 1;
      const int qbase = 128 * q_tile(i) + 64 * w;
      const bool need_mask = (CAUSAL && qbase + p.off < k0 + 127) || (qbase + 64 > p.N) ||
                             (k0 + 128 > p.N_kv);
      // Phase 1: P = 2^(S scale log2e - lse log2e), kept in registers (fp32) and written to
      // TMEM as bf16 pairs over the first half of this warpgroup's S^T columns.
      ok = warp_wait(bar(L::bQFull + st), ph, abort_flag) &&
           warp_wait(bar(L::bSFull), i & 1, abort_flag);
      if (!ok) break;
      tc_fence_after();
      const float* lse2 = reinterpret_cast<const float*>(gbase + L::kRow + st * 1024) + 64 * w;
      float pr[64];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t s[32];
        tmem_ld_32x32b_x32(tmem + L::tS + 64 * w + 32 * h + lane_off, s);
        tmem_ld_wait();
        reg_fence(s);
#pragma unroll
        for (int c = 0; c < 32; c += 4) {
          const float4 l4 = *reinterpret_cast<const float4*>(lse2 + 32 * h + c);
          float a[4];
          f2_unpack(f2_fma(f2_pack_u(s[c], s[c + 1]), sl2x2, f2_pack(l4.x, l4.y)), a[0], a[1]);
          f2_unpack(f2_fma(f2_pack_u(s[c + 2], s[c + 3]), sl2x2, f2_pack(l4.z, l4.w)), a[2],
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
        for (int c = 0; c < 16; ++c) pk[c] = pack_bf16x2(pr[32 * h + 2 * c], pr[32 * h + 2 * c + 1]);
        tmem_st_32x32b_x16(tmem + L::tS + 64 * w + 16 * h + lane_off, pk);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(L::bPDone));
      // Phase 2: dS = P o (dP - D) to shared memory (bf16, K-major for dK's A operand and
      // MN-major for dQ^T's B operand), once dK(i-1) and dQ(i-1) have read the previous one.
      ok = warp_wait(bar(L::bDPFull), i & 1, abort_flag) &&
           (i == 0 || warp_wait(bar(L::bDQFull), (i - 1) & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      const float* Dv = reinterpret_cast<const float*>(gbase + L::kRow + st * 1024 + 512) + 64 * w;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t dp[32];
        tmem_ld_32x32b_x32(tmem + L::tDP + 64 * w + 32 * h + lane_off, dp);
        tmem_ld_wait();
        reg_fence(dp);
        uint32_t dsk[16];
#pragma unroll
        for (int c = 0; c < 32; c += 4) {
          const float4 d4 = *reinterpret_cast<const float4*>(Dv + 32 * h + c);
          float dsr[4];
          f2_unpack(f2_mul(f2_pack(pr[32 * h + c], pr[32 * h + c + 1]),
                           f2_sub(f2_pack_u(dp[c], dp[c + 1]), f2_pack(d4.x, d4.y))),
                    dsr[0], dsr[1]);
          f2_unpack(f2_mul(f2_pack(pr[32 * h + c + 2], pr[32 * h + c + 3]),
                           f2_sub(f2_pack_u(dp[c + 2], dp[c + 3]), f2_pack(d4.z, d4.w))),
                    dsr[2], dsr[3]);
          dsk[c / 2] = pack_bf16x2(dsr[0], dsr[1]);
          dsk[c / 2 + 1] = pack_bf16x2(dsr[2], dsr[3]);
        }
#pragma unroll
        for (int t = 0; t < 4; ++t)
          *reinterpret_cast<uint4*>(dsb + sw128_offset(r, 4 * h + t)) =
              make_uint4(dsk[4 * t], dsk[4 * t + 1], dsk[4 * t + 2], dsk[4 * t + 3]);
        // and to TMEM over this warpgroup's first dP^T columns, already read (h = 0 writes
        // columns 64w .. 64w+15, below the ones h = 1 reads): the A operand of dK
        tmem_st_32x32b_x16(tmem + L::tDP + 64 * w + 16 * h + lane_off, dsk);
      }
      tmem_st_wait();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar(L::bDSDone));
    }
    if (!ok) fail(p.status, abort_flag, 5);
    // ------------------------------------------------------------ dV / dK epilogue -------
    if (ok && (n_i == 0 || warp_wait(bar(L::bAccDone), 0, abort_flag))) {
      tc_fence_after();
      // warpgroup 0 stores dV (stage-0 Q space), warpgroup 1 stores dK * scale (stage-1 Q)
      const uint32_t tcol = w == 0 ? L::tDV : L::tDK;
      const float mul = w == 0 ? 1.0f : p.scale;
      const int region = L::kQ + w * L::kTile;
      uint8_t* stage = gbase + region;
#pragma unroll
      for (int c = 0; c < D; c += 32) {
        uint32_t v[32];
        if (n_i > 0) {
          tmem_ld_32x32b_x32(tmem + tcol + c + lane_off, v);
          tmem_ld_wait();
          reg_fence(v);
        } else {  // no query sees these keys: dK = dV = 0 (TMEM was never written)
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = 0u;
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint4 u;
          u.x = pack_bf16x2(__uint_as_float(v[8 * q + 0]) * mul, __uint_as_float(v[8 * q + 1]) * mul);
          u.y = pack_bf16x2(__uint_as_float(v[8 * q + 2]) * mul, __uint_as_float(v[8 * q + 3]) * mul);
          u.z = pack_bf16x2(__uint_as_float(v[8 * q + 4]) * mul, __uint_as_float(v[8 * q + 5]) * mul);
          u.w = pack_bf16x2(__uint_as_float(v[8 * q + 6]) * mul, __uint_as_float(v[8 * q + 7]) * mul);
          const int chunk = c / 8 + q;
          *reinterpret_cast<uint4*>(stage + (chunk >> 3) * L::kBox + sw128_offset(r, chunk & 7)) = u;
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        const CUtensorMap* map = w == 0 ? &tmDV : &tmDK;
#pragma unroll
        for (int bx = 0; bx < L::kBoxes; ++bx)
          tma_store_3d(map, sbase + region + bx * L::kBox + (warp & 3) * 4096, 64 * bx,
                       k0 + (warp & 3) * 32, bh);
        bulk_commit_group();
        bulk_wait_group_read0();
      }
    } else if (ok) {
      fail(p.status, abort_flag, 5);
    }
  } else if (warp < 12 && D == 64) {
    // ------------------------------------------------------- dQ drain (d = 64) ----------
    // dQ(i) sits in TMEM as [128 queries (lanes)][64 columns]: warp wq holds queries
    // [32 wq, 32 wq + 32) of the tile and stages them as two 32 x 32 fp32 boxes in the 128-byte
    // swizzled layout (16-byte stores, conflict-free), each added into the accumulator by one
    // TMA reduction.
    bwd128_setmaxnreg<R::kDrain>();
    const int wq = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const float scale = p.scale;
    uint8_t* stageb = gbase + L::kDQ + wq * 8192;
    const uint32_t stage_s = sbase + L::kDQ + wq * 8192;
    bool ok = true;
    for (int i = 0; i < n_i; ++i) {
      if (!warp_wait(bar(L::bDQFull), i & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      uint32_t v[64];
#pragma unroll
      for (int c = 0; c < 2; ++c)
        tmem_ld_32x32b_x32(tmem + L::tDP + 32 * c + lane_off,
                           *reinterpret_cast<uint32_t(*)[32]>(&v[32 * c]));
      tmem_ld_wait();
      reg_fence(v);
      tc_fence_before();
      mbar_arrive(bar(L::bDQFree));
      const int q0 = 128 * q_tile(i) + 32 * wq, qh = q_head(i);
      if (q0 >= p.N) continue;  // no rows of this warp's slice exist
      if (lane == 0) bulk_wait_group_read0();  // the previous reduction has read the staging
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
        tma_reduce_add_3d(&tmDQacc, stage_s, 0, q0, qh);
        tma_reduce_add_3d(&tmDQacc, stage_s + 4096, 32, q0, qh);
        bulk_commit_group();
      }
    }
    if (!ok) fail(p.status, abort_flag, 5);
    if (lane == 0) bulk_wait_group0();
  } else if (warp < 12) {
    // ------------------------------------------------------ dQ drain (d = 128) ----------
    bwd128_setmaxnreg<R::kDrain>();
    const int wq = warp & 3;                        // dQ^T rows (d) [32 wq, 32 wq + 32)
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const bool active = 32 * wq < p.d;              // rows past d (d = 96) are zero
    const float scale = p.scale;
    float* stagef = reinterpret_cast<float*>(gbase + L::kDQ + wq * 8192);
    const uint32_t stage_s = sbase + L::kDQ + wq * 8192;
    bool ok = true;
    for (int i = 0; i < n_i; ++i) {
      if (!warp_wait(bar(L::bDQFull), i & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      // all of dQ^T(i) into registers first, so the MMA can reuse the columns at once
      uint32_t v[128];
#pragma unroll
      for (int c = 0; c < 4; ++c)
        tmem_ld_32x32b_x32(tmem + L::tDP + 32 * c + lane_off,
                           *reinterpret_cast<uint32_t(*)[32]>(&v[32 * c]));
      tmem_ld_wait();
      reg_fence(v);
      tc_fence_before();
      mbar_arrive(bar(L::bDQFree));
      if (!active) continue;
      const int q0 = 128 * q_tile(i), qh = q_head(i);
#pragma unroll
      for (int hq = 0; hq < 2; ++hq) {
        if (q0 + 64 * hq >= p.N) break;  // no rows of this half exist
        if (lane == 0) bulk_wait_group_read0();  // the previous reduction has read the staging
        __syncwarp();
        // staging box: 64 query rows x 32 columns (this warp's d slice), fp32
#pragma unroll
        for (int q = 0; q < 64; ++q) stagef[q * 32 + lane] = __uint_as_float(v[64 * hq + q]) * scale;
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_reduce_add_3d(&tmDQacc, stage_s, 32 * wq, q0 + 64 * hq, qh);
          bulk_commit_group();
        }
      }
    }
    if (!ok) fail(p.status, abort_flag, 5);
    if (lane == 0) bulk_wait_group0();
  } else {
    bwd128_setmaxnreg<R::kOther>();
    if (warp == 12 && lane == 0) {
      // ------------------------------------------------------------------- MMA ----------
      const uint32_t id_s = idesc_bf16_f32(128, 128, false, false);  // S^T, dP^T
      const uint32_t id_acc = idesc_bf16_f32(128, D, false, true);   // dV, dK
      const uint32_t id_dq = idesc_bf16_f32(128, 128 * D / 128, true, true);  // dQ^T, or dQ
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
      auto mma_s = [&](int i) {  // S^T = K Q^T
        const uint32_t so = static_cast<uint32_t>(i & 1) * L::kTile;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_ss(tmem + L::tS, sdesc_advance(dK_k, kmaj(kk)), sdesc_advance(dQ_k, so + kmaj(kk)),
                  id_s, kk > 0 ? 1u : 0u);
      };
      auto mma_dp = [&]() {  // dP^T = V dO^T
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_ss(tmem + L::tDP, sdesc_advance(dV_k, kmaj(kk)), sdesc_advance(dDO_k, kmaj(kk)),
                  id_s, kk > 0 ? 1u : 0u);
      };
      auto mma_dv = [&](int i) {  // dV += P^T dO; P^T from TMEM (warpgroup w's queries at 64w)
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_ts(tmem + L::tDV, tmem + L::tS + (kk >> 2) * 64 + (kk & 3) * 8,
                  sdesc_advance(dDO_mn, kk * 2048), id_acc, (kk > 0 || i > 0) ? 1u : 0u);
      };
      auto mma_dk = [&](int i) {  // dK += dS^T Q; dS^T from TMEM (its bf16 copy over dP^T)
        const uint32_t so = static_cast<uint32_t>(i & 1) * L::kTile;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_ts(tmem + L::tDK, tmem + L::tDP + (kk >> 2) * 64 + (kk & 3) * 8,
                  sdesc_advance(dQ_mn, so + kk * 2048), id_acc, (kk > 0 || i > 0) ? 1u : 0u);
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
      bool ok = n_i == 0 || mbar_wait(bar(L::bKV), 0, abort_flag, lim);
      for (int i = 0; i <= n_i && ok; ++i) {
        const int st = i & 1;
        const uint32_t ph = (i >> 1) & 1;
        if (i < n_i) {
          if (!(ok = mbar_wait(bar(L::bQFull + st), ph, abort_flag, lim))) break;
          tc_fence_after();
          mma_s(i);
          umma_commit(bar(L::bSFull));
        }
        if (i > 0) {
          if (!(ok = mbar_wait(bar(L::bDSDone), (i - 1) & 1, abort_flag, lim))) break;
          tc_fence_after();
          mma_dk(i - 1);
          umma_commit(bar(L::bQEmpty + ((i - 1) & 1)));
          mma_dq();
          umma_commit(bar(L::bDQFull));
        }
        if (i < n_i) {
          if (!(ok = mbar_wait(bar(L::bOFull), i & 1, abort_flag, lim) &&
                     mbar_wait(bar(L::bPDone), i & 1, abort_flag, lim)))
            break;
          tc_fence_after();
          mma_dv(i);
          if (i > 0) {
            if (!(ok = mbar_wait(bar(L::bDQFree), (i - 1) & 1, abort_flag, lim))) break;
            tc_fence_after();
          }
          mma_dp();
          umma_commit(bar(L::bDPFull));
          umma_commit(bar(L::bOEmpty));
        }
      }
      if (ok && n_i > 0) umma_commit(bar(L::bAccDone));
      if (!ok) fail(p.status, abort_flag, 5);
      // Every MMA this thread issued completes before tensor memory is freed (the drain after a
      // give-up; on the normal path the epilogue waits for the same products). Bounded wait.
      volatile int never = 0;
      umma_commit(bar(L::bDrain));
      mbar_wait(bar(L::bDrain), 0, &never);
    } else if (warp == 13 && lane == 0) {
      // ------------------------------------------------------------------- TMA ----------
      if (n_i > 0) {
        mbar_arrive_expect_tx(bar(L::bKV), 2 * L::kTile);
#pragma unroll
        for (int bx = 0; bx < L::kBoxes; ++bx) {
          tma_load_3d(sbase + L::kK + bx * L::kBox, &tmK, bar(L::bKV), 64 * bx, k0, bh);
          tma_load_3d(sbase + L::kV + bx * L::kBox, &tmV, bar(L::bKV), 64 * bx, k0, bh);
        }
      }
      int issued_o = 0, issued_q = 0;
      for (int i = 0; i < n_i; ++i) {
        const int st = i & 1;
        const int q0 = 128 * q_tile(i), qh = q_head(i);
        const uint32_t so = static_cast<uint32_t>(st) * L::kTile;
        // Q(i) with its row terms: the stage frees after dK(i-2)
        if (!mbar_wait(bar(L::bQEmpty + st), ((i >> 1) & 1) ^ 1, abort_flag)) {
          fail(p.status, abort_flag, 5);
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
        }
        issued_q = i + 1;
        // dO(i): the single slot frees after dP(i-1)
        if (i > 0 && !mbar_wait(bar(L::bOEmpty), (i - 1) & 1, abort_flag)) {
          fail(p.status, abort_flag, 5);
          break;
        }
        mbar_arrive_expect_tx(bar(L::bOFull), L::kTile);
#pragma unroll
        for (int bx = 0; bx < L::kBoxes; ++bx)
          tma_load_3d(sbase + L::kDO + bx * L::kBox, &tmDO, bar(L::bOFull), 64 * bx, q0, qh);
        issued_o = i + 1;
      }
      // Every load issued lands before the CTA can exit, whether or not (or whenever) a role
      // gives up; these are the latest loads of their slots, so on the normal path the bounded
      // waits return at once.
      volatile int never = 0;
      if (issued_o > 0) mbar_wait(bar(L::bOFull), (issued_o - 1) & 1, &never);
      for (int i = max(0, issued_q - 2); i < issued_q; ++i)
        if (i != p.dbg_skip) mbar_wait(bar(L::bQFull + (i & 1)), (i >> 1) & 1, &never);
      if (n_i > 0) mbar_wait(bar(L::bKV), 0, &never);
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

// fa_bwd_d256.cuh — exact attention backward for head dimension 256 on sm_100a.
//
// The mathematics of fa_bwd.cuh ("How FlashAttention Actually Works", section "The Backward
// Pass: Recomputation": S and P are recomputed on chip from Q, K and the stored logsumexp):
//     P = exp(S - lse),  dV = P^T dO,  dP = dO V^T,  D_i = dO_i . O_i,  dS = P o (dP - D),
//     dQ = scale dS K,   dK = scale dS^T Q,
// with the same preprocess (D, -lse log2e, dQ accumulator zeroed) and dQ conversion kernels.
//
// At d = 256 the fp32 accumulators of a 128-key tile, dK and dV, are 256 TMEM columns each:
// together they fill all 512, leaving none for S^T and dP^T. The main work is therefore split
// into two passes over the same (key/value head, 128-key tile) grid, each keeping one of the
// two accumulators:
//   pass 1, fa_bwd_d256_dv:   S^T = K Q^T -> P^T (TMEM, in place) -> dV += P^T dO
//       TMEM: dV [0,256), two S^T buffers [256,320) and [320,384) (64 queries each), so the
//       tensor core computes S^T(i+1) and dV(i) while the elementwise warps work on S^T(i).
//       SMEM: K (64 KB), a 2-stage ring of Q tiles and of dO tiles (32 KB each) with the
//       tile's -lse log2e.
//   pass 2, fa_bwd_d256_dkdq: S^T, dP^T = V dO^T -> dS^T (SMEM) -> dK += dS^T Q and
//       dQ^T = K^T dS^T (two 128-row halves of d) -> TMA bulk reduction into dQ_acc
//       TMEM: dK [0,256), S^T [256,320), dP^T [320,384), dQ^T [384,512).
//       SMEM: K, V (64 KB each), one Q and one dO tile (32 KB each), dS^T (16 KB), dQ staging
//       (16 KB), the tile's -lse log2e and D.
// Query tiles are 64 rows, so S^T, dP^T and dQ^T are M = 128, N = 64 products and dV, dK are
// M = 128, N = 256 products; S^T is computed in both passes (6 products per tile pair instead
// of 5), the price of fitting TMEM.
//
// Roles (16 warps): warps 0-7 elementwise (thread = key row, warpgroup w = queries
// 32w .. 32w+31 of the tile; then the dV or dK epilogue), warps 8-11 dQ drain (pass 2),
// warp 12 MMA issue, warp 13 TMA.
#pragma once
#include "fa_bwd.cuh"

namespace fa {

struct Bwd256Geom {
  static constexpr int kKVBox = 128 * 128;  // TMA box: 128 rows x 64 bf16 columns (SW128)
  static constexpr int kQBox = 64 * 128;    // TMA box: 64 rows x 64 bf16 columns
  static constexpr int kKVTile = 4 * kKVBox;  // 128 x 256 bf16 = 64 KB
  static constexpr int kQTile = 4 * kQBox;    // 64 x 256 bf16 = 32 KB
};

struct Bwd256DvLayout : Bwd256Geom {
  static constexpr int kK = 0;
  static constexpr int kQ = kKVTile;                // + stage * kQTile (2 stages); dV staging
  static constexpr int kDO = kQ + 2 * kQTile;       // + stage * kQTile
  static constexpr int kRow = kDO + 2 * kQTile;     // + stage * 256: -lse log2e of 64 queries
  static constexpr int kBars = kRow + 2 * 256;
  static constexpr int bKV = 0, bQFull = 1, bQEmpty = 3, bOFull = 5, bOEmpty = 7;  // + stage
  static constexpr int bSFull = 9;                  // + buffer
  static constexpr int bPDone = 11;                 // + buffer (256 arrivals)
  static constexpr int bAccDone = 13, bDrain = 14, kNumBars = 15;
  static constexpr int kTmemSlot = kBars + kNumBars * 8;
  static constexpr int kBytes = kTmemSlot + 8;
  static constexpr int kAlloc = kBytes + 1024;      // slack for the 1024-byte alignment
  static constexpr uint32_t tDV = 0;
  __host__ __device__ static constexpr uint32_t tS(int b) { return 256u + 64u * b; }
};
static_assert(Bwd256DvLayout::kAlloc + 16 <= 227 * 1024, "d = 256 dV pass shared memory");

struct Bwd256DkdqLayout : Bwd256Geom {
  static constexpr int kK = 0;
  static constexpr int kV = kKVTile;
  static constexpr int kQ = 2 * kKVTile;            // one slot; with dO, the dK staging
  static constexpr int kDO = kQ + kQTile;
  static constexpr int kDS = kDO + kQTile;          // dS^T [128 keys][64 queries] bf16, SW128
  static constexpr int kDQ = kDS + 16384;           // dQ staging: 4 warps x (32 x 32 fp32)
  static constexpr int kRow = kDQ + 16384;          // -lse log2e [64], then D [64]
  static constexpr int kBars = kRow + 512;
  static constexpr int bKV = 0, bQFull = 1, bQEmpty = 2, bOFull = 3, bOEmpty = 4;
  static constexpr int bSFull = 5, bDPFull = 6;
  static constexpr int bSPRead = 7;                 // S^T, dP^T loaded to registers (256)
  static constexpr int bDSDone = 8;                 // dS^T in shared memory (256 arrivals)
  static constexpr int bDSFree = 9;                 // dK and dQ^T have read dS^T
  static constexpr int bDQFull = 10;                // dQ^T in TMEM
  static constexpr int bDQFree = 11;                // dQ^T copied out of TMEM (128 arrivals)
  static constexpr int bAccDone = 12, bDrain = 13, kNumBars = 14;
  static constexpr int kTmemSlot = kBars + kNumBars * 8;
  static constexpr int kBytes = kTmemSlot + 8;
  static constexpr int kAlloc = kBytes + 1024;
  static constexpr uint32_t tDK = 0, tS = 256, tDP = 320, tDQ = 384;  // tDQ + 64 h for half h
};
static_assert(Bwd256DkdqLayout::kAlloc + 16 <= 227 * 1024, "d = 256 dK/dQ pass shared memory");

// Work unit and query-tile iteration shared by both passes: the scheduling of fa_bwd_main
// (L2-sized groups of key/value heads, key tiles with the most query tiles first).
struct Bwd256Unit {
  int bh, k0, qi0, n_qt, n_i, qgroup;
  __device__ Bwd256Unit(const BwdParams& p, bool causal) {
    int j;
    grouped_unit(static_cast<int>(blockIdx.x), p.n_kv, p.BH_kv, p.group, j, bh);
    k0 = 128 * j;
    qi0 = causal ? max(0, k0 - p.off) / 64 : 0;  // first 64-row tile that sees this key tile
    n_qt = max(0, p.n_q - qi0);
    qgroup = p.qgroup;
    n_i = qgroup * n_qt;
  }
  __device__ int q_head(int it) const { return bh * qgroup + it / n_qt; }
  __device__ int q_tile(int it) const { return qi0 + it % n_qt; }
};

// Columns c (0..31) of a 32-query slice starting at qbase that key `key` may not see: c < lo or
// c >= hi. Returns false when none is masked (the common case), so callers can skip the pass.
template <bool CAUSAL>
__device__ __forceinline__ bool bwd256_mask(const BwdParams& p, int qbase, int key, int& lo,
                                            int& hi) {
  lo = CAUSAL ? key - p.off - qbase : 0;
  hi = p.N - qbase;
  if (key >= p.N_kv) lo = 32;
  return lo > 0 || hi < 32;
}

// dV or dK (x mul) of a 128-key tile from TMEM columns [tcol, tcol + 256) to global memory:
// warp w8 (0..7) of the elementwise warps converts columns [128 (w8 / 4), +128) of its 32 rows
// to bf16 in the 64 KB staging area (four 128 x 64 boxes) and stores its two boxes with TMA.
__device__ __forceinline__ void bwd256_store_acc(uint32_t tmem_acc, bool have, float mul,
                                                 uint8_t* stage, uint32_t stage_s,
                                                 const CUtensorMap* map, int k0, int bh,
                                                 int warp, int lane) {
  const int w = warp >> 2, r4 = warp & 3, row = 32 * r4 + lane;
  const uint32_t lane_off = static_cast<uint32_t>(32 * r4) << 16;
#pragma unroll
  for (int c = 0; c < 128; c += 32) {
    uint32_t v[32];
    if (have) {
      tmem_ld_32x32b_x32(tmem_acc + 128 * w + c + lane_off, v);
      tmem_ld_wait();
      reg_fence(v);
    } else {  // no query sees these keys: the gradient is exactly zero
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
      const int chunk = (128 * w + c) / 8 + q;  // 0 .. 31: box chunk / 8, 16-byte chunk % 8
      *reinterpret_cast<uint4*>(stage + (chunk >> 3) * Bwd256Geom::kKVBox +
                                sw128_offset(row, chunk & 7)) = u;
    }
  }
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
#pragma unroll
    for (int bx = 2 * w; bx < 2 * w + 2; ++bx)
      tma_store_3d(map, stage_s + bx * Bwd256Geom::kKVBox + r4 * 4096, 64 * bx, k0 + 32 * r4, bh);
    bulk_commit_group();
    bulk_wait_group_read0();
  }
}

// S^T = K Q^T for one 64-query tile: M = 128 keys, N = 64 queries, K = 256 (16 k-steps).
__device__ __forceinline__ void bwd256_mma_st(uint32_t d_tmem, uint64_t k_desc, uint64_t q_desc) {
  const uint32_t id = idesc_bf16_f32(128, 64, false, false);
#pragma unroll
  for (int kk = 0; kk < 16; ++kk)
    umma_ss(d_tmem,
            sdesc_advance(k_desc, static_cast<uint32_t>((kk >> 2) * Bwd256Geom::kKVBox + (kk & 3) * 32)),
            sdesc_advance(q_desc, static_cast<uint32_t>((kk >> 2) * Bwd256Geom::kQBox + (kk & 3) * 32)),
            id, kk > 0 ? 1u : 0u);
}

// ============================================================================================
// Pass 1: dV.
// ============================================================================================
template <bool CAUSAL>
__global__ void __launch_bounds__(kBwdThreads, 1)
    fa_bwd_d256_dv(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmDO,
                   const __grid_constant__ CUtensorMap tmLse2,
                   const __grid_constant__ CUtensorMap tmDV, const BwdParams p) {
  using L = Bwd256DvLayout;
  extern __shared__ uint8_t smem_raw[];
  __shared__ int abort_flag_storage;
  volatile int* abort_flag = &abort_flag_storage;
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (sbase - raw);
  auto bar = [&](int i) -> uint32_t { return sbase + L::kBars + 8u * i; };
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const Bwd256Unit u(p, CAUSAL);
  const int n_i = u.n_i;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(bar(L::bKV), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(L::bQFull + s), 1);
      mbar_init(bar(L::bQEmpty + s), 1);
      mbar_init(bar(L::bOFull + s), 1);
      mbar_init(bar(L::bOEmpty + s), 1);
      mbar_init(bar(L::bSFull + s), 1);
      mbar_init(bar(L::bPDone + s), 256);
    }
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
    tma_prefetch_desc(&tmDO);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(gbase + L::kTmemSlot);

  if (warp < 8) {
    // --------------------------------------------------------- P^T (elementwise) --------
    const int w = warp >> 2;                       // queries [32w, 32w+32) of the tile
    const int r = threadIdx.x & 127;               // key row (TMEM lane)
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int key = u.k0 + r;
    const uint64_t sl2x2 = f2_pack(p.scale_log2, p.scale_log2);
    bool ok = true;
    for (int i = 0; i < n_i && ok; ++i) {
      const int b = i & 1;
      const uint32_t ph = (i >> 1) & 1;
      // the row terms travel with dO(i), whose stage is refilled only after dV(i)
      ok = warp_wait(bar(L::bOFull + b), ph, abort_flag) &&
           warp_wait(bar(L::bSFull + b), ph, abort_flag);
      if (!ok) break;
      tc_fence_after();
      uint32_t s[32];
      tmem_ld_32x32b_x32(tmem + L::tS(b) + 32 * w + lane_off, s);
      tmem_ld_wait();
      reg_fence(s);
      const float* lse2 = reinterpret_cast<const float*>(gbase + L::kRow + b * 256) + 32 * w;
      const int qbase = 64 * u.q_tile(i) + 32 * w;
      float pr[32];
#pragma unroll
      for (int c = 0; c < 32; c += 4) {
        const float4 l4 = *reinterpret_cast<const float4*>(lse2 + c);
        float a[4];
        f2_unpack(f2_fma(f2_pack_u(s[c], s[c + 1]), sl2x2, f2_pack(l4.x, l4.y)), a[0], a[1]);
        f2_unpack(f2_fma(f2_pack_u(s[c + 2], s[c + 3]), sl2x2, f2_pack(l4.z, l4.w)), a[2], a[3]);
#pragma unroll
        for (int e = 0; e < 4; ++e) pr[c + e] = ex2_approx(a[e]);
      }
      int lo, hi;
      if (bwd256_mask<CAUSAL>(p, qbase, key, lo, hi)) {
#pragma unroll
        for (int c = 0; c < 32; ++c)
          if (c < lo || c >= hi) pr[c] = 0.f;
      }
      uint32_t pk[16];
#pragma unroll
      for (int c = 0; c < 16; ++c) pk[c] = pack_bf16x2(pr[2 * c], pr[2 * c + 1]);
      // in place, over this warpgroup's own first 16 columns of S^T
      tmem_st_32x32b_x16(tmem + L::tS(b) + 32 * w + lane_off, pk);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(L::bPDone + b));
    }
    if (ok && (n_i == 0 || warp_wait(bar(L::bAccDone), 0, abort_flag))) {
      tc_fence_after();
      bwd256_store_acc(tmem + L::tDV, n_i > 0, 1.0f, gbase + L::kQ, sbase + L::kQ, &tmDV, u.k0,
                       u.bh, warp, lane);
    } else {
      fail(p.status, abort_flag, 5);
    }
  } else if (warp == 12) {
    if (lane == 0) {
      // ------------------------------------------------------------------ MMA ------------
      const uint64_t lim = p.limit_ns;
      const uint64_t dK_k = sdesc_sw128(sbase + L::kK, 16, 1024);                // K-major
      const uint64_t dQ_k = sdesc_sw128(sbase + L::kQ, 16, 1024);                // K-major
      const uint64_t dDO_mn = sdesc_sw128(sbase + L::kDO, L::kQBox, 1024);       // MN-major
      const uint32_t id_dv = idesc_bf16_f32(128, 256, false, true);
      auto issue_s = [&](int i) {  // S^T(i) into buffer i % 2; frees Q stage i % 2 when done
        const int b = i & 1;
        bwd256_mma_st(tmem + L::tS(b), dK_k, sdesc_advance(dQ_k, b * L::kQTile));
        umma_commit(bar(L::bSFull + b));
        umma_commit(bar(L::bQEmpty + b));
      };
      bool ok = n_i == 0 || mbar_wait(bar(L::bKV), 0, abort_flag, lim);
      for (int i = 0; i < 2 && i < n_i && ok; ++i) {
        if (!(ok = mbar_wait(bar(L::bQFull + i), 0, abort_flag, lim))) break;
        tc_fence_after();
        issue_s(i);
      }
      for (int i = 0; i < n_i && ok; ++i) {
        const int b = i & 1;
        const uint32_t ph = (i >> 1) & 1;
        if (!(ok = mbar_wait(bar(L::bPDone + b), ph, abort_flag, lim))) break;
        tc_fence_after();
        // dV += P^T dO: A = P^T from TMEM (queries 16kk.. of warpgroup kk / 2 at its columns
        // 32 (kk / 2) + 8 (kk % 2)), B = dO, MN-major, N = 256
        const uint64_t o0 = sdesc_advance(dDO_mn, b * L::kQTile);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_ts(tmem + L::tDV, tmem + L::tS(b) + (kk >> 1) * 32 + (kk & 1) * 8,
                  sdesc_advance(o0, kk * 2048), id_dv, (kk > 0 || i > 0) ? 1u : 0u);
        umma_commit(bar(L::bOEmpty + b));
        if (i + 2 < n_i) {  // S^T(i+2) reuses buffer b after dV(i) (products run in order)
          if (!(ok = mbar_wait(bar(L::bQFull + b), ph ^ 1, abort_flag, lim))) break;
          tc_fence_after();
          issue_s(i + 2);
        }
      }
      if (ok && n_i > 0) umma_commit(bar(L::bAccDone));
      if (!ok) fail(p.status, abort_flag, 5);
      volatile int never = 0;
      umma_commit(bar(L::bDrain));
      mbar_wait(bar(L::bDrain), 0, &never);
    }
  } else if (warp == 13) {
    if (lane == 0) {
      // ------------------------------------------------------------------ TMA ------------
      if (n_i > 0) {
        mbar_arrive_expect_tx(bar(L::bKV), L::kKVTile);
#pragma unroll
        for (int bx = 0; bx < 4; ++bx)
          tma_load_3d(sbase + L::kK + bx * L::kKVBox, &tmK, bar(L::bKV), 64 * bx, u.k0, u.bh);
      }
      int issued_q = 0, issued_o = 0;
      for (int i = 0; i < n_i; ++i) {
        const int st = i & 1;
        const uint32_t ph = ((i >> 1) & 1) ^ 1;
        const int q0 = 64 * u.q_tile(i), qh = u.q_head(i);
        if (!mbar_wait(bar(L::bQEmpty + st), ph, abort_flag)) {
          fail(p.status, abort_flag, 5);
          break;
        }
        if (i != p.dbg_skip) {  // (the test hook leaves this tile out)
          mbar_arrive_expect_tx(bar(L::bQFull + st), L::kQTile);
#pragma unroll
          for (int bx = 0; bx < 4; ++bx)
            tma_load_3d(sbase + L::kQ + st * L::kQTile + bx * L::kQBox, &tmQ,
                        bar(L::bQFull + st), 64 * bx, q0, qh);
        }
        issued_q = i + 1;
        if (!mbar_wait(bar(L::bOEmpty + st), ph, abort_flag)) {
          fail(p.status, abort_flag, 5);
          break;
        }
        mbar_arrive_expect_tx(bar(L::bOFull + st), L::kQTile + 256);
#pragma unroll
        for (int bx = 0; bx < 4; ++bx)
          tma_load_3d(sbase + L::kDO + st * L::kQTile + bx * L::kQBox, &tmDO,
                      bar(L::bOFull + st), 64 * bx, q0, qh);
        tma_load_3d(sbase + L::kRow + st * 256, &tmLse2, bar(L::bOFull + st), q0, qh, 0);
        issued_o = i + 1;
      }
      // Every load issued lands before the CTA can exit (on the normal path these bounded
      // waits return at once: they are the latest loads of their stages).
      volatile int never = 0;
      for (int i = max(0, issued_q - 2); i < issued_q; ++i)
        if (i != p.dbg_skip) mbar_wait(bar(L::bQFull + (i & 1)), (i >> 1) & 1, &never);
      for (int i = max(0, issued_o - 2); i < issued_o; ++i)
        mbar_wait(bar(L::bOFull + (i & 1)), (i >> 1) & 1, &never);
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

// ============================================================================================
// Pass 2: dK and dQ.
// ============================================================================================
template <bool CAUSAL>
__global__ void __launch_bounds__(kBwdThreads, 1)
    fa_bwd_d256_dkdq(const __grid_constant__ CUtensorMap tmQ,
                     const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV,
                     const __grid_constant__ CUtensorMap tmDO,
                     const __grid_constant__ CUtensorMap tmLse2,
                     const __grid_constant__ CUtensorMap tmD,
                     const __grid_constant__ CUtensorMap tmDQacc,
                     const __grid_constant__ CUtensorMap tmDK, const BwdParams p) {
  using L = Bwd256DkdqLayout;
  extern __shared__ uint8_t smem_raw[];
  __shared__ int abort_flag_storage;
  volatile int* abort_flag = &abort_flag_storage;
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (sbase - raw);
  auto bar = [&](int i) -> uint32_t { return sbase + L::kBars + 8u * i; };
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const Bwd256Unit u(p, CAUSAL);
  const int n_i = u.n_i;

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(bar(L::bKV), 1);
    mbar_init(bar(L::bQFull), 1);
    mbar_init(bar(L::bQEmpty), 1);
    mbar_init(bar(L::bOFull), 1);
    mbar_init(bar(L::bOEmpty), 1);
    mbar_init(bar(L::bSFull), 1);
    mbar_init(bar(L::bDPFull), 1);
    mbar_init(bar(L::bSPRead), 256);
    mbar_init(bar(L::bDSDone), 256);
    mbar_init(bar(L::bDSFree), 1);
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
    // ------------------------------------------------------ dS^T (elementwise) ----------
    const int w = warp >> 2;                       // queries [32w, 32w+32) of the tile
    const int r = threadIdx.x & 127;               // key row (TMEM lane)
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int key = u.k0 + r;
    const uint64_t sl2x2 = f2_pack(p.scale_log2, p.scale_log2);
    bool ok = true;
    for (int i = 0; i < n_i && ok; ++i) {
      const uint32_t ph = i & 1;
      ok = warp_wait(bar(L::bQFull), ph, abort_flag) &&
           warp_wait(bar(L::bSFull), ph, abort_flag) &&
           warp_wait(bar(L::bDPFull), ph, abort_flag);
      if (!ok) break;
      tc_fence_after();
      uint32_t s[32], dp[32];
      tmem_ld_32x32b_x32(tmem + L::tS + 32 * w + lane_off, s);
      tmem_ld_32x32b_x32(tmem + L::tDP + 32 * w + lane_off, dp);
      tmem_ld_wait();
      reg_fence(s);
      reg_fence(dp);
      tc_fence_before();
      mbar_arrive(bar(L::bSPRead));  // S^T(i+1), dP^T(i+1) may now overwrite both regions
      const float* lse2 = reinterpret_cast<const float*>(gbase + L::kRow) + 32 * w;
      const float* Dv = reinterpret_cast<const float*>(gbase + L::kRow + 256) + 32 * w;
      const int qbase = 64 * u.q_tile(i) + 32 * w;
      uint32_t dsk[16];
#pragma unroll
      for (int c = 0; c < 32; c += 4) {
        const float4 l4 = *reinterpret_cast<const float4*>(lse2 + c);
        const float4 d4 = *reinterpret_cast<const float4*>(Dv + c);
        float a[4], pr[4], dsr[4];
        f2_unpack(f2_fma(f2_pack_u(s[c], s[c + 1]), sl2x2, f2_pack(l4.x, l4.y)), a[0], a[1]);
        f2_unpack(f2_fma(f2_pack_u(s[c + 2], s[c + 3]), sl2x2, f2_pack(l4.z, l4.w)), a[2], a[3]);
#pragma unroll
        for (int e = 0; e < 4; ++e) pr[e] = ex2_approx(a[e]);
        f2_unpack(f2_mul(f2_pack(pr[0], pr[1]),
                         f2_sub(f2_pack_u(dp[c], dp[c + 1]), f2_pack(d4.x, d4.y))),
                  dsr[0], dsr[1]);
        f2_unpack(f2_mul(f2_pack(pr[2], pr[3]),
                         f2_sub(f2_pack_u(dp[c + 2], dp[c + 3]), f2_pack(d4.z, d4.w))),
                  dsr[2], dsr[3]);
        dsk[c / 2] = pack_bf16x2(dsr[0], dsr[1]);
        dsk[c / 2 + 1] = pack_bf16x2(dsr[2], dsr[3]);
      }
      int lo, hi;
      if (bwd256_mask<CAUSAL>(p, qbase, key, lo, hi)) {
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const uint32_t keep_lo = (c < lo || c >= hi) ? 0u : 0x0000ffffu;
          const uint32_t keep_hi = (c + 1 < lo || c + 1 >= hi) ? 0u : 0xffff0000u;
          dsk[c / 2] &= keep_lo | keep_hi;
        }
      }
      // dS^T(i-1) has been read by dK(i-1) and dQ^T(i-1) before this one is written
      if (i > 0 && !(ok = warp_wait(bar(L::bDSFree), (i - 1) & 1, abort_flag))) break;
      uint8_t* dsb = gbase + L::kDS;
#pragma unroll
      for (int t = 0; t < 4; ++t)
        *reinterpret_cast<uint4*>(dsb + sw128_offset(r, 4 * w + t)) =
            make_uint4(dsk[4 * t], dsk[4 * t + 1], dsk[4 * t + 2], dsk[4 * t + 3]);
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar(L::bDSDone));
    }
    if (ok && (n_i == 0 || warp_wait(bar(L::bAccDone), 0, abort_flag))) {
      tc_fence_after();
      // staging: the Q and dO slots (64 KB), no longer read once every product has completed
      bwd256_store_acc(tmem + L::tDK, n_i > 0, p.scale, gbase + L::kQ, sbase + L::kQ, &tmDK,
                       u.k0, u.bh, warp, lane);
    } else {
      fail(p.status, abort_flag, 5);
    }
  } else if (warp < 12) {
    // ---------------------------------------------------------------- dQ drain ----------
    const int wq = warp & 3;  // rows 32 wq .. 32 wq + 31 of each 128-row half of d
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    float* stagef = reinterpret_cast<float*>(gbase + L::kDQ + wq * 4096);
    const uint32_t stage_s = sbase + L::kDQ + wq * 4096;
    bool ok = true;
    for (int i = 0; i < n_i; ++i) {
      if (!warp_wait(bar(L::bDQFull), i & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      const int q0 = 64 * u.q_tile(i), qh = u.q_head(i);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t v[64];
        tmem_ld_32x32b_x32(tmem + L::tDQ + 64 * h + lane_off, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
        tmem_ld_32x32b_x32(tmem + L::tDQ + 64 * h + 32 + lane_off,
                           *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
        tmem_ld_wait();
        reg_fence(v);
        if (h == 1) {  // both halves are in registers: the next dQ^T may overwrite them
          tc_fence_before();
          mbar_arrive(bar(L::bDQFree));
        }
#pragma unroll
        for (int qq = 0; qq < 2; ++qq) {  // 32-query quarters of the tile
          if (q0 + 32 * qq >= p.N) break;  // no rows of this quarter exist
          if (lane == 0) bulk_wait_group_read0();  // the previous reduction read the staging
          __syncwarp();
#pragma unroll
          for (int q = 0; q < 32; ++q)
            stagef[q * 32 + lane] = __uint_as_float(v[32 * qq + q]) * p.scale;
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_reduce_add_3d(&tmDQacc, stage_s, 128 * h + 32 * wq, q0 + 32 * qq, qh);
            bulk_commit_group();
          }
        }
      }
    }
    if (!ok) fail(p.status, abort_flag, 5);
    if (lane == 0) bulk_wait_group0();
  } else if (warp == 12) {
    if (lane == 0) {
      // ------------------------------------------------------------------ MMA ------------
      const uint64_t lim = p.limit_ns;
      const uint64_t dK_k = sdesc_sw128(sbase + L::kK, 16, 1024);                // K-major
      const uint64_t dV_k = sdesc_sw128(sbase + L::kV, 16, 1024);                // K-major
      const uint64_t dQ_k = sdesc_sw128(sbase + L::kQ, 16, 1024);                // K-major
      const uint64_t dDO_k = sdesc_sw128(sbase + L::kDO, 16, 1024);              // K-major
      const uint64_t dQ_mn = sdesc_sw128(sbase + L::kQ, L::kQBox, 1024);         // MN-major
      const uint64_t dDS_k = sdesc_sw128(sbase + L::kDS, 16, 1024);              // dS^T K-major
      const uint64_t dDS_mn = sdesc_sw128(sbase + L::kDS, 16, 1024);             // dS^T MN-major
      const uint64_t dKt_mn = sdesc_sw128(sbase + L::kK, L::kKVBox, 1024);       // K^T MN-major
      const uint32_t id_dk = idesc_bf16_f32(128, 256, false, true);
      const uint32_t id_dq = idesc_bf16_f32(128, 64, true, true);
      auto issue_s = [&]() {
        bwd256_mma_st(tmem + L::tS, dK_k, dQ_k);
        umma_commit(bar(L::bSFull));
      };
      auto issue_dp = [&]() {  // dP^T = V dO^T; dO's slot is free once this has completed
        bwd256_mma_st(tmem + L::tDP, dV_k, dDO_k);
        umma_commit(bar(L::bDPFull));
        umma_commit(bar(L::bOEmpty));
      };
      bool ok = n_i == 0 || mbar_wait(bar(L::bKV), 0, abort_flag, lim);
      if (ok && n_i > 0) {
        ok = mbar_wait(bar(L::bQFull), 0, abort_flag, lim) &&
             mbar_wait(bar(L::bOFull), 0, abort_flag, lim);
        if (ok) {
          tc_fence_after();
          issue_s();
          issue_dp();
        }
      }
      for (int i = 0; i < n_i && ok; ++i) {
        const uint32_t ph = i & 1;
        // dP^T(i+1) as soon as the elementwise warps hold dP^T(i) and dO(i+1) has landed
        if (i + 1 < n_i) {
          if (!(ok = mbar_wait(bar(L::bSPRead), ph, abort_flag, lim) &&
                     mbar_wait(bar(L::bOFull), ph ^ 1, abort_flag, lim)))
            break;
          tc_fence_after();
          issue_dp();
        }
        if (!(ok = mbar_wait(bar(L::bDSDone), ph, abort_flag, lim))) break;
        tc_fence_after();
        // dK += dS^T Q: A = dS^T (K-major), B = Q (MN-major, N = 256). Q(i) is then free.
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_ss(tmem + L::tDK, sdesc_advance(dDS_k, kk * 32), sdesc_advance(dQ_mn, kk * 2048),
                  id_dk, (kk > 0 || i > 0) ? 1u : 0u);
        umma_commit(bar(L::bQEmpty));
        if (i > 0 && !(ok = mbar_wait(bar(L::bDQFree), ph ^ 1, abort_flag, lim))) break;
        tc_fence_after();
        // dQ^T = K^T dS^T, one M = 128 product per half of d: A = K^T (MN-major; the half's
        // two 64-column boxes of K), B = dS^T (MN-major, N = 64)
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_ss(tmem + L::tDQ + 64 * h, sdesc_advance(dKt_mn, 2 * h * L::kKVBox + kk * 2048),
                    sdesc_advance(dDS_mn, kk * 2048), id_dq, kk > 0 ? 1u : 0u);
        umma_commit(bar(L::bDQFull));
        umma_commit(bar(L::bDSFree));
        if (i + 1 < n_i) {  // S^T(i+1) once Q(i+1) is in (its slot was freed by dK(i))
          if (!(ok = mbar_wait(bar(L::bQFull), ph ^ 1, abort_flag, lim))) break;
          tc_fence_after();
          issue_s();
        }
      }
      if (ok && n_i > 0) umma_commit(bar(L::bAccDone));
      if (!ok) fail(p.status, abort_flag, 5);
      volatile int never = 0;
      umma_commit(bar(L::bDrain));
      mbar_wait(bar(L::bDrain), 0, &never);
    }
  } else if (warp == 13) {
    if (lane == 0) {
      // ------------------------------------------------------------------ TMA ------------
      if (n_i > 0) {
        mbar_arrive_expect_tx(bar(L::bKV), 2 * L::kKVTile);
#pragma unroll
        for (int bx = 0; bx < 4; ++bx) {
          tma_load_3d(sbase + L::kK + bx * L::kKVBox, &tmK, bar(L::bKV), 64 * bx, u.k0, u.bh);
          tma_load_3d(sbase + L::kV + bx * L::kKVBox, &tmV, bar(L::bKV), 64 * bx, u.k0, u.bh);
        }
      }
      int issued_q = 0, issued_o = 0;
      for (int i = 0; i < n_i; ++i) {
        const uint32_t ph = (i & 1) ^ 1;
        const int q0 = 64 * u.q_tile(i), qh = u.q_head(i);
        // dO(i) and Q(i) with its row terms; the slots free after dP(i-1) and dK(i-1)
        if (!mbar_wait(bar(L::bOEmpty), ph, abort_flag)) {
          fail(p.status, abort_flag, 5);
          break;
        }
        mbar_arrive_expect_tx(bar(L::bOFull), L::kQTile);
#pragma unroll
        for (int bx = 0; bx < 4; ++bx)
          tma_load_3d(sbase + L::kDO + bx * L::kQBox, &tmDO, bar(L::bOFull), 64 * bx, q0, qh);
        issued_o = i + 1;
        if (!mbar_wait(bar(L::bQEmpty), ph, abort_flag)) {
          fail(p.status, abort_flag, 5);
          break;
        }
        if (i != p.dbg_skip) {  // (the test hook leaves this tile out)
          mbar_arrive_expect_tx(bar(L::bQFull), L::kQTile + 512);
#pragma unroll
          for (int bx = 0; bx < 4; ++bx)
            tma_load_3d(sbase + L::kQ + bx * L::kQBox, &tmQ, bar(L::bQFull), 64 * bx, q0, qh);
          tma_load_3d(sbase + L::kRow, &tmLse2, bar(L::bQFull), q0, qh, 0);
          tma_load_3d(sbase + L::kRow + 256, &tmD, bar(L::bQFull), q0, qh, 0);
        }
        issued_q = i + 1;
      }
      // Every load issued lands before the CTA can exit (on the normal path these bounded
      // waits return at once: they are the latest loads of their slots).
      volatile int never = 0;
      if (issued_o > 0) mbar_wait(bar(L::bOFull), (issued_o - 1) & 1, &never);
      if (issued_q > 0 && issued_q - 1 != p.dbg_skip)
        mbar_wait(bar(L::bQFull), (issued_q - 1) & 1, &never);
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

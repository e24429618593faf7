// fa_fwd_d256.cuh — exact attention forward for head dimension 256 on sm_100a.
//
// The computation of fa_fwd.cuh ("How FlashAttention Actually Works", sections "How Tiling
// Works" and "The Secret Weapon: Online Softmax") with 256-column Q, K, V rows. The two-tile
// layout of the d <= 128 kernel does not fit: two 128 x 256 fp32 O accumulators alone would
// take all 512 TMEM columns. Here one CTA owns one 128-row query tile and keeps two S buffers
// instead, so the tensor core computes S(j+1) and O += P(j) V(j) while the softmax works on S(j):
//   TMEM: S0 [0,128), S1 [128,256), O [256,512).
//   SMEM: Q 64 KB (reused as O staging), a two-slot ring of 64 KB K / V tiles.
// MMA issue order: S(0); then per key tile j: S(j+1), PV(j). The ring holds the tiles in the
// same order (K0, K1, V0, K2, V1, ...). P (bf16) is written over the first 64 columns of its S
// buffer and read by the PV MMA straight from TMEM.
//
// Roles (16 warps): warps 0-3 softmax (one thread per row), warps 4-7 idle (their registers go
// to the softmax), warps 8-11 epilogue, warp 12 MMA, warp 13 TMA.
#pragma once
#include "fa_fwd.cuh"
#include "sm100.cuh"

namespace fa {

struct Fwd256Layout {
  static constexpr int kBoxBytes = 128 * 64 * 2;    // one TMA box: 128 rows x 64 bf16 columns
  static constexpr int kBoxes = 4;                  // 256 columns
  static constexpr int kTileBytes = 128 * 256 * 2;  // 64 KB
  static constexpr int kStages = 2;
  static constexpr int kQ = 0;
  static constexpr int kKV = kTileBytes;
  static constexpr int kBars = kKV + kStages * kTileBytes;
  static constexpr int bQ = 0;
  static constexpr int bKvFull = 1;                 // + slot
  static constexpr int bKvEmpty = 1 + kStages;      // + slot
  static constexpr int bSFull = 1 + 2 * kStages;    // + S buffer
  static constexpr int bPFull = bSFull + 2;         // + S buffer (128 arrivals)
  static constexpr int bODone = bPFull + 2;         // one completion per PV
  static constexpr int bFinal = bODone + 1;         // 128 arrivals
  static constexpr int bDrain = bFinal + 1;         // error path only
  static constexpr int kNumBars = bDrain + 1;
  static constexpr int kRowL = kBars + kNumBars * 8;
  static constexpr int kTmemSlot = kRowL + 128 * 4;
  static constexpr int kBytes = kTmemSlot + 16;
  static constexpr int kAlloc = kBytes + 1024;
};
static_assert(Fwd256Layout::kAlloc <= 227 * 1024, "d = 256 forward shared memory");

// Register split (setmaxnreg, per warpgroup): the idle warpgroup gives its registers to the
// softmax; the four shares must add up to the launch allocation (512 threads x 128).
struct Fwd256Regs {
  static constexpr uint32_t kLaunch = 128;  // registers per thread at launch (checked on the host)
  static constexpr uint32_t kSoftmax = 232, kIdle = 24, kEpilogue = 104, kMma = 152;
  static_assert(128 * (kSoftmax + kIdle + kEpilogue + kMma) == kFwdThreads * kLaunch,
                "d = 256 forward register split must equal the launch allocation");
};

// Moves this warp's register allocation from the launch value to R: setmaxnreg.inc when R is
// larger, setmaxnreg.dec when smaller (each direction only accepts its own kind of change).
template <uint32_t R>
__device__ __forceinline__ void setmaxnreg_to() {
  static_assert(R % 8 == 0 && R >= 24 && R <= 256, "setmaxnreg range");
  if constexpr (R > Fwd256Regs::kLaunch)
    setmaxnreg_inc<R>();
  else if constexpr (R < Fwd256Regs::kLaunch)
    setmaxnreg_dec<R>();
}

template <bool CAUSAL>
__global__ void __launch_bounds__(kFwdThreads, 1)
    fa_fwd_d256_kernel(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV,
                       const __grid_constant__ CUtensorMap tmO, const FwdParams p) {
  using L = Fwd256Layout;
  using R = Fwd256Regs;
  constexpr int ST = L::kStages;
  constexpr int D = 256;
  extern __shared__ uint8_t smem_raw[];
  __shared__ int abort_flag_storage;
  volatile int* abort_flag = &abort_flag_storage;

  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (sbase - raw);
  auto bar = [&](int i) -> uint32_t { return sbase + L::kBars + 8u * i; };
  float* s_rowl = reinterpret_cast<float*>(gbase + L::kRowL);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // L2-sized head groups, longest first inside a group, as in fa_fwd.cuh
  int qb, bh;
  fwd_work_unit(static_cast<int>(blockIdx.x), p.n_qblocks, p.BH, p.hgroup, qb, bh);
  const int bh_kv = bh / p.group;
  const int q0 = qb * 128;
  const int nkv = (p.N_kv + 127) / 128;
  const int last_key = q0 + 127 + p.off;
  const int n = !CAUSAL ? nkv : (last_key < 0 ? 0 : min(nkv, last_key / 128 + 1));

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(bar(L::bQ), 1);
    for (int s = 0; s < ST; ++s) {
      mbar_init(bar(L::bKvFull + s), 1);
      mbar_init(bar(L::bKvEmpty + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(L::bSFull + b), 1);
      mbar_init(bar(L::bPFull + b), 128);
    }
    mbar_init(bar(L::bODone), 1);
    mbar_init(bar(L::bFinal), 128);
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
    tma_prefetch_desc(&tmO);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(gbase + L::kTmemSlot);

  if (warp >= 4 && warp < 8) {
    setmaxnreg_to<R::kIdle>();
  } else if (warp < 4) {
    setmaxnreg_to<R::kSoftmax>();
    {
      // ---------------------------------------------------------------- softmax ----------
      const int row = threadIdx.x & 127;
      const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
      const int q_row = q0 + row;
      const float sl2 = p.scale_log2;
      float m = -INFINITY, l = 0.f, lr = 0.f;
      for (int j = 0; j < n; ++j) {
        const int b = j & 1;
        const uint32_t tS = tmem + b * 128 + lane_off;
        if (!warp_wait(bar(L::bSFull + b), (j >> 1) & 1, abort_flag)) {
          fail(p.status, abort_flag, 5);
          break;
        }
        tc_fence_after();
        uint32_t s[128];
        tmem_ld_32x32b_x32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
        tmem_ld_32x32b_x32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
        tmem_ld_32x32b_x32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(&s[64]));
        tmem_ld_32x32b_x32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(&s[96]));
        tmem_ld_wait();
        reg_fence(s);
        const int kv0 = j * 128;
        if ((CAUSAL && kv0 + 127 > q0 + p.off) || (kv0 + 128 > p.N_kv)) {
          const int lim = CAUSAL ? min(q_row + 1 + p.off, p.N_kv) : p.N_kv;
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (kv0 + c >= lim) s[c] = __float_as_uint(-INFINITY);
        }
        // columns 0-7 seed the four running maxima; the loop takes 8 columns per step up to 127
        float mx0 = fmaxf(__uint_as_float(s[0]), __uint_as_float(s[4]));
        float mx1 = fmaxf(__uint_as_float(s[1]), __uint_as_float(s[5]));
        float mx2 = fmaxf(__uint_as_float(s[2]), __uint_as_float(s[6]));
        float mx3 = fmaxf(__uint_as_float(s[3]), __uint_as_float(s[7]));
#pragma unroll
        for (int c = 8; c < 128; c += 8) {
          mx0 = max3f(mx0, __uint_as_float(s[c]), __uint_as_float(s[c + 1]));
          mx1 = max3f(mx1, __uint_as_float(s[c + 2]), __uint_as_float(s[c + 3]));
          mx2 = max3f(mx2, __uint_as_float(s[c + 4]), __uint_as_float(s[c + 5]));
          mx3 = max3f(mx3, __uint_as_float(s[c + 6]), __uint_as_float(s[c + 7]));
        }
        // threshold update of the running max, exact as in fa_fwd.cuh
        const float m_tile = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3));
        float alpha = 1.0f;
        if ((m_tile - m) * sl2 > kRescaleLog2) {
          alpha = ex2_approx((m - m_tile) * sl2);
          m = m_tile;
        }
        const float nb = m == -INFINITY ? 0.f : -m * sl2;
        const uint64_t sl2x2 = f2_pack(sl2, sl2), nbx2 = f2_pack(nb, nb);
        uint64_t lsum[4] = {0, 0, 0, 0}, rsum[4] = {0, 0, 0, 0};
        uint32_t pk[64];
#pragma unroll
        for (int c = 0; c < 128; c += 2) {
          float a0, a1;
          f2_unpack(f2_fma(f2_pack_u(s[c], s[c + 1]), sl2x2, nbx2), a0, a1);
          const float e0 = ex2_approx(a0), e1 = ex2_approx(a1);
          const uint32_t w = pack_bf16x2(e0, e1);
          pk[c / 2] = w;
          lsum[(c >> 1) & 3] = f2_add(lsum[(c >> 1) & 3], f2_pack(e0, e1));
          rsum[(c >> 1) & 3] = f2_add(rsum[(c >> 1) & 3], f2_pack_u(w << 16, w & 0xffff0000u));
        }
        {
          const uint64_t ls = f2_add(f2_add(lsum[0], lsum[1]), f2_add(lsum[2], lsum[3]));
          const uint64_t rs = f2_add(f2_add(rsum[0], rsum[1]), f2_add(rsum[2], rsum[3]));
          float x0, x1, y0, y1;
          f2_unpack(ls, x0, x1);
          f2_unpack(rs, y0, y1);
          l = l * alpha + (x0 + x1);
          lr = lr * alpha + (y0 + y1);
        }
        tmem_st_32x32b_x32(tS + 0, *reinterpret_cast<const uint32_t(*)[32]>(&pk[0]));
        tmem_st_32x32b_x32(tS + 32, *reinterpret_cast<const uint32_t(*)[32]>(&pk[32]));
        // O correction. S(j) may complete before PV(j-1) (it was issued first), so the warp
        // waits for PV(j-1) — the j-th completion of bODone — before touching O (rare: only
        // when some row's running max rose).
        if (j > 0 && __any_sync(0xffffffffu, alpha != 1.0f)) {
          if (!warp_wait(bar(L::bODone), (j - 1) & 1, abort_flag)) {
            fail(p.status, abort_flag, 5);
            break;
          }
          tc_fence_after();
          const uint32_t tO = tmem + 256 + lane_off;
#pragma unroll 1
          for (int c = 0; c < D; c += 32) {
            uint32_t o[32];
            tmem_ld_32x32b_x32(tO + c, o);
            tmem_ld_wait();
            reg_fence(o);
            const uint64_t a2 = f2_pack(alpha, alpha);
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
              const uint64_t r = f2_mul(f2_pack_u(o[i], o[i + 1]), a2);
              o[i] = static_cast<uint32_t>(r);
              o[i + 1] = static_cast<uint32_t>(r >> 32);
            }
            tmem_st_32x32b_x32(tO + c, o);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(bar(L::bPFull + b));
      }
      s_rowl[row] = lr;
      mbar_arrive(bar(L::bFinal));
      if (!*abort_flag && q_row < p.N)
        p.lse[static_cast<size_t>(bh) * p.N + q_row] =
            l > 0.f ? (m * sl2 + lg2_approx(l)) * 0.69314718055994531f : -INFINITY;
    }
  } else if (warp < 12) {
    // ----------------------------------------------------------------- epilogue ----------
    setmaxnreg_to<R::kEpilogue>();
    const int row = threadIdx.x - 256;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    // O / lr -> bf16 -> swizzled staging in the Q tile -> TMA; each warp stores its 32 rows.
    // With no key tile there is no MMA ordering the staging after the Q load: wait for it.
    if (warp_wait(bar(L::bFinal), 0, abort_flag) &&
        (n == 0 || warp_wait(bar(L::bODone), (n - 1) & 1, abort_flag)) &&
        (n > 0 || warp_wait(bar(L::bQ), 0, abort_flag))) {
      tc_fence_after();
      const float lr_row = s_rowl[row];
      const float inv_l = lr_row > 0.f ? 1.0f / lr_row : 0.f;
      const uint32_t tO = tmem + 256 + lane_off;
      uint8_t* stage = gbase + L::kQ;
#pragma unroll 1
      for (int c = 0; c < D; c += 32) {
        uint32_t o[32];
        if (n > 0) {
          tmem_ld_32x32b_x32(tO + c, o);
          tmem_ld_wait();
          reg_fence(o);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0u;
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint4 v;
          v.x = pack_bf16x2(__uint_as_float(o[8 * q + 0]) * inv_l, __uint_as_float(o[8 * q + 1]) * inv_l);
          v.y = pack_bf16x2(__uint_as_float(o[8 * q + 2]) * inv_l, __uint_as_float(o[8 * q + 3]) * inv_l);
          v.z = pack_bf16x2(__uint_as_float(o[8 * q + 4]) * inv_l, __uint_as_float(o[8 * q + 5]) * inv_l);
          v.w = pack_bf16x2(__uint_as_float(o[8 * q + 6]) * inv_l, __uint_as_float(o[8 * q + 7]) * inv_l);
          const int chunk = c / 8 + q;  // 0 .. 31
          *reinterpret_cast<uint4*>(stage + (chunk >> 3) * L::kBoxBytes +
                                    sw128_offset(row, chunk & 7)) = v;
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
#pragma unroll
        for (int b = 0; b < L::kBoxes; ++b)
          tma_store_3d(&tmO, sbase + L::kQ + b * L::kBoxBytes + (warp & 3) * 4096, 64 * b,
                       q0 + (warp & 3) * 32, bh);
        bulk_commit_group();
        bulk_wait_group_read0();
      }
    } else {
      fail(p.status, abort_flag, 5);
    }
  } else {
    setmaxnreg_to<R::kMma>();
    if (warp == 12 && lane == 0) {
      // ------------------------------------------------------------------ MMA -------------
      const uint32_t idesc_qk = idesc_bf16_f32(128, 128, false, false);
      const uint32_t idesc_pv = idesc_bf16_f32(128, D, false, true);
      const uint64_t desc_q = sdesc_sw128(sbase + L::kQ, 16, 1024);              // K-major
      const uint64_t desc_k0 = sdesc_sw128(sbase + L::kKV, 16, 1024);            // K-major
      const uint64_t desc_v0 = sdesc_sw128(sbase + L::kKV, L::kBoxBytes, 1024);  // MN-major
      int u = 0;  // ring position of the next tile, in the producer's order
      auto wait_full = [&](int uu) -> bool {
        return mbar_wait(bar(L::bKvFull + uu % ST), (uu / ST) & 1, abort_flag);
      };
      auto issue_s = [&](int j) {  // S(j) from the K tile at ring position u
        const uint64_t b0 = sdesc_advance(desc_k0, (u % ST) * L::kTileBytes);
        const uint32_t d = tmem + (j & 1) * 128;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * L::kBoxBytes + (kk & 3) * 32;
          umma_ss(d, sdesc_advance(desc_q, off), sdesc_advance(b0, off), idesc_qk, kk > 0 ? 1u : 0u);
        }
        umma_commit(bar(L::bSFull + (j & 1)));
        umma_commit(bar(L::bKvEmpty + u % ST));
        ++u;
      };
      auto issue_pv = [&](int j) {  // O += P(j) V(j), V at ring position u
        const uint64_t b0 = sdesc_advance(desc_v0, (u % ST) * L::kTileBytes);
        const uint32_t a = tmem + (j & 1) * 128;
        umma_ts(tmem + 256, a, b0, idesc_pv, j > 0 ? 1u : 0u);
#pragma unroll
        for (int kk = 1; kk < 8; ++kk)
          umma_ts(tmem + 256, a + kk * 8, sdesc_advance(b0, kk * 2048), idesc_pv, 1u);
        umma_commit(bar(L::bODone));
        umma_commit(bar(L::bKvEmpty + u % ST));
        ++u;
      };
      bool ok = n == 0 || (mbar_wait(bar(L::bQ), 0, abort_flag) && wait_full(u));
      if (ok && n > 0) {
        tc_fence_after();
        issue_s(0);
      }
      for (int j = 0; j < n && ok; ++j) {
        if (j + 1 < n) {
          // S(j+1) goes to the buffer that held P(j-1), read by PV(j-1), issued earlier
          if (!wait_full(u)) { ok = false; break; }
          tc_fence_after();
          issue_s(j + 1);
        }
        if (!mbar_wait(bar(L::bPFull + (j & 1)), (j >> 1) & 1, abort_flag) || !wait_full(u)) {
          ok = false;
          break;
        }
        tc_fence_after();
        issue_pv(j);
      }
      if (!ok) {
        fail(p.status, abort_flag, 5);
        volatile int never = 0;
        umma_commit(bar(L::bDrain));
        mbar_wait(bar(L::bDrain), 0, &never);
      }
    } else if (warp == 13 && lane == 0) {
      // ------------------------------------------------------------------ TMA -------------
      mbar_arrive_expect_tx(bar(L::bQ), L::kTileBytes);
#pragma unroll
      for (int b = 0; b < L::kBoxes; ++b)
        tma_load_3d(sbase + L::kQ + b * L::kBoxBytes, &tmQ, bar(L::bQ), 64 * b, q0, bh);
      // ring order: K0, then per key tile j: K(j+1) (if any), V(j)
      int issued = 0;
      bool ok = true;
      auto load = [&](const CUtensorMap* map, int j) -> bool {
        const int st = issued % ST;
        if (!mbar_wait(bar(L::bKvEmpty + st), ((issued / ST) & 1) ^ 1, abort_flag)) return false;
        mbar_arrive_expect_tx(bar(L::bKvFull + st), L::kTileBytes);
        const uint32_t dst = sbase + L::kKV + st * L::kTileBytes;
#pragma unroll
        for (int b = 0; b < L::kBoxes; ++b)
          tma_load_3d(dst + b * L::kBoxBytes, map, bar(L::bKvFull + st), 64 * b, 128 * j, bh_kv);
        ++issued;
        return true;
      };
      if (n > 0) ok = load(&tmK, 0);
      for (int j = 0; j < n && ok; ++j) {
        if (j + 1 < n) ok = load(&tmK, j + 1);
        if (ok) ok = load(&tmV, j);
      }
      if (!ok) fail(p.status, abort_flag, 5);
      if (*abort_flag || n == 0) {
        // let the loads in flight land before shared memory is released
        volatile int never = 0;
        for (int uu = max(0, issued - ST); uu < issued; ++uu)
          mbar_wait(bar(L::bKvFull + uu % ST), (uu / ST) & 1, &never);
        mbar_wait(bar(L::bQ), 0, &never);
      }
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

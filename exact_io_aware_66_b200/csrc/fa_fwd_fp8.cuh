// fa_fwd_fp8.cuh — exact attention forward with FP8 (E4M3) Q, K, V on sm_100a.
//
// The same tiled online-softmax forward as fa_fwd.cuh ("How FlashAttention Actually Works",
// sections "How Tiling Works" and "The Secret Weapon: Online Softmax"), with 8-bit operands:
// "How does FlashAttention optimize memory and speed via tiling?", section "Interview tips",
// names FP8 as a feature of a later version. Q, K and V arrive as E4M3 codes, each tensor with
// an fp32 descale factor; both products run on tcgen05.mma kind::f8f6f4 (E4M3 x E4M3, fp32
// accumulation in TMEM). S = Q K^T is exact in fp32 (products of E4M3 values are exact); the
// probabilities P are rounded to E4M3 for the PV product, and O is normalised by the sum of
// exactly those rounded weights. O is written in bf16, lse in fp32 from the unrounded sum.
//
// Layout: one internal head dimension of 128 bytes per row (d = 64 or 96 is zero-extended by
// the TMA loads). The PV product wants V with the key index contiguous (K-major B operand), so
// V is first transposed into a workspace [B*H_kv][d][N_kv padded to 16] by fa_fp8_transpose_v.
//
// Roles (16 warps), TMEM, the issue order and the persistent scheduling (cluster launch control,
// units handed to the roles through a two-slot ring, barrier phases counted over the CTA's
// run) are those of fa_fwd.cuh; P takes 32 TMEM columns (four E4M3 per column) at the start of
// its S buffer.
#pragma once
#include <cuda_fp8.h>

#include "fa_fwd.cuh"
#include "sm100.cuh"

namespace fa {

struct Fp8Layout {
  static constexpr int kTile = 128 * 128;         // 128 rows x 128 bytes (one swizzle span)
  static constexpr int kOBoxBytes = 128 * 64 * 2;  // bf16 O store box: 128 rows x 64 columns
  static constexpr int kOTile = 128 * 128 * 2;     // bf16 O tile staging
  static constexpr int kStages = 6;                // K / V^T ring
  static constexpr int kQ = 0;                     // Q0, Q1
  static constexpr int kKV = 2 * kTile;
  static constexpr int kO = kKV + kStages * kTile;  // O0, O1 staging
  static constexpr int kBars = kO + 2 * kOTile;
  static constexpr int kNumBars = 1 + 2 * kStages + 19;
  static constexpr int kRowL = kBars + kNumBars * 8;
  static constexpr int kSched = kRowL + 2 * 128 * 4;       // two unit indices
  static constexpr int kClc = (kSched + 8 + 15) / 16 * 16;  // 16-byte launch-control reply
  static constexpr int kTmemSlot = kClc + 16;
  static constexpr int kBytes = kTmemSlot + 16;
  static constexpr int kAlloc = kBytes + 1024;

  // barriers as in FwdLayout
  static constexpr int bQ = 0;
  static constexpr int bKvFull = 1;
  static constexpr int bKvEmpty = 1 + kStages;
  static constexpr int bSFull = 1 + 2 * kStages;
  static constexpr int bPFull = bSFull + 2;
  static constexpr int bODone = bSFull + 4;
  static constexpr int bFinal = bSFull + 6;
  static constexpr int bOFree = bSFull + 8;
  static constexpr int bRowFree = bSFull + 10;
  static constexpr int bSchedFull = bSFull + 12;
  static constexpr int bSchedEmpty = bSFull + 14;
  static constexpr int bQEmpty = bSFull + 16;
  static constexpr int bClc = bSFull + 17;
  static constexpr int bDrain = bSFull + 18;
  static constexpr int kSchedReaders = 13;
};
static_assert(Fp8Layout::kAlloc <= 227 * 1024, "fp8 forward shared memory");

struct Fp8Params {
  float* lse;
  int* status;
  int N, N_kv, BH, group, off, n_qblocks;
  int hgroup;        // query heads per scheduling group (fwd_work_unit)
  int o_boxes;       // 64-column boxes of O actually stored: ceil(d / 64)
  float scale_log2;  // softmax scale * log2(e) * q_descale * k_descale
  float o_scale;     // v_descale
};

// Instruction descriptor for tcgen05.mma kind::f8f6f4 with E4M3 A and B (format code 0), fp32
// accumulation, both operands K-major (PTX ISA, "Instruction descriptor": [4,6) D format,
// [7,10) A format, [10,13) B format, [17,23) N >> 3, [24,29) M >> 4).
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N) {
  return (1u << 4) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void umma_ss_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// A from TMEM: row m in lane m, four E4M3 per 32-bit column (element k in byte k % 4 of
// column k / 4).
__device__ __forceinline__ void umma_ts_f8(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Rounds (a, b) to E4M3 (nearest even, saturating at 448) into the low and high byte of a
// 16-bit word, and returns the rounded values widened back to fp32.
__device__ __forceinline__ uint32_t e4m3x2_round(float a, float b, float& ra, float& rb) {
  const __nv_fp8x2_storage_t s = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE,
                                                          __NV_E4M3);
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(s, __NV_E4M3);
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h));
  ra = f.x;
  rb = f.y;
  return static_cast<uint32_t>(s);
}

template <bool CAUSAL>
__global__ void __launch_bounds__(kFwdThreads, 1)
    fa_fwd_fp8_kernel(const __grid_constant__ CUtensorMap tmQ,
                      const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmVt,
                      const __grid_constant__ CUtensorMap tmO, const Fp8Params p) {
  using L = Fp8Layout;
  using R = FwdRegs<128, false>;
  constexpr int ST = L::kStages;
  extern __shared__ uint8_t smem_raw[];
  __shared__ int abort_flag_storage;
  volatile int* abort_flag = &abort_flag_storage;

  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (sbase - raw);
  auto bar = [&](int i) -> uint32_t { return sbase + L::kBars + 8u * i; };
  float* s_rowl = reinterpret_cast<float*>(gbase + L::kRowL);
  volatile int* sched = reinterpret_cast<volatile int*>(gbase + L::kSched);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nkv = (p.N_kv + 127) / 128;
  struct Unit {  // as in fa_fwd_kernel
    int q0, bh, n_t[2];
  };
  auto unit_of = [&](int u) {
    Unit w;
    int qb;
    fwd_work_unit(u, p.n_qblocks, p.BH, p.hgroup, qb, w.bh);
    w.q0 = qb * 256;
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int last_key = w.q0 + 128 * t + 127 + p.off;
      w.n_t[t] = !CAUSAL ? nkv : (last_key < 0 ? 0 : min(nkv, last_key / 128 + 1));
    }
    return w;
  };

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(bar(L::bQ), 1);
    for (int s = 0; s < ST; ++s) {
      mbar_init(bar(L::bKvFull + s), 1);
      mbar_init(bar(L::bKvEmpty + s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(L::bSFull + t), 1);
      mbar_init(bar(L::bPFull + t), 128);
      mbar_init(bar(L::bODone + t), 1);
      mbar_init(bar(L::bFinal + t), 128);
      mbar_init(bar(L::bOFree + t), 128);
      mbar_init(bar(L::bRowFree + t), 128);
      mbar_init(bar(L::bSchedFull + t), 1);
      mbar_init(bar(L::bSchedEmpty + t), L::kSchedReaders);
    }
    mbar_init(bar(L::bQEmpty), 1);
    mbar_init(bar(L::bClc), 1);
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
    tma_prefetch_desc(&tmVt);
    tma_prefetch_desc(&tmO);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(gbase + L::kTmemSlot);

  constexpr int kGaveUp = -2;
  auto warp_next_unit = [&](int s) -> int {
    if (!warp_wait(bar(L::bSchedFull + (s & 1)), (s >> 1) & 1, abort_flag)) return kGaveUp;
    const int u = sched[s & 1];
    __syncwarp();
    if (lane == 0) mbar_arrive(bar(L::bSchedEmpty + (s & 1)));
    return u;
  };

  if (warp < 8) {
    // ------------------------------------------------------------------ softmax ----------
    setmaxnreg_inc<R::kSoftmax>();
    const int t = warp >> 2;
    const int row = threadIdx.x & 127;
    const uint32_t tS = tmem + t * 128 + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const float sl2 = p.scale_log2;
    int sc = 0;  // S tiles of this query tile in earlier units
    bool ok = true;
    for (int si = 0, uc = 0; ok; ++si, ++uc) {
      const int u = warp_next_unit(si);
      if (u == kGaveUp) { ok = false; break; }
      if (u < 0) break;
      const Unit U = unit_of(u);
      const int q0 = U.q0, bh = U.bh, n = U.n_t[t];
      const int q_row = q0 + t * 128 + row;
      float m = -INFINITY;
      float l = 0.f;   // sum of the fp32 exponentials: gives lse
      float lr = 0.f;  // sum of the same exponentials rounded to E4M3: normalises O
      for (int j = 0; j < n; ++j) {
        if (!warp_wait(bar(L::bSFull + t), (sc + j) & 1, abort_flag)) {
          ok = false;
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
        const bool need_mask = (CAUSAL && kv0 + 127 > q0 + t * 128 + p.off) || (kv0 + 128 > p.N_kv);
        if (need_mask) {
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
        // Threshold update of the running max as in fa_fwd.cuh: weights stay below 2^8, inside
        // E4M3's range (448).
        const float m_tile = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3));
        float alpha = 1.0f;
        if ((m_tile - m) * sl2 > kRescaleLog2) {
          alpha = ex2_approx((m - m_tile) * sl2);
          m = m_tile;
        }
        const float nb = m == -INFINITY ? 0.f : -m * sl2;
        const uint64_t sl2x2 = f2_pack(sl2, sl2), nbx2 = f2_pack(nb, nb);
        uint64_t lsum[2] = {0, 0}, rsum[2] = {0, 0};
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 128; c += 4) {
          float a0, a1, a2, a3;
          f2_unpack(f2_fma(f2_pack_u(s[c], s[c + 1]), sl2x2, nbx2), a0, a1);
          f2_unpack(f2_fma(f2_pack_u(s[c + 2], s[c + 3]), sl2x2, nbx2), a2, a3);
          const float e0 = ex2_approx(a0), e1 = ex2_approx(a1);
          const float e2 = ex2_approx(a2), e3 = ex2_approx(a3);
          float r0, r1, r2, r3;
          const uint32_t lo = e4m3x2_round(e0, e1, r0, r1);
          const uint32_t hi = e4m3x2_round(e2, e3, r2, r3);
          pk[c / 4] = lo | (hi << 16);
          const int acc = (c >> 2) & 1;
          lsum[acc] = f2_add(lsum[acc], f2_add(f2_pack(e0, e1), f2_pack(e2, e3)));
          rsum[acc] = f2_add(rsum[acc], f2_add(f2_pack(r0, r1), f2_pack(r2, r3)));
        }
        {
          const uint64_t ls = f2_add(lsum[0], lsum[1]);
          const uint64_t rs = f2_add(rsum[0], rsum[1]);
          float x0, x1, y0, y1;
          f2_unpack(ls, x0, x1);
          f2_unpack(rs, y0, y1);
          l = l * alpha + (x0 + x1);
          lr = lr * alpha + (y0 + y1);
        }
        tmem_st_32x32b_x32(tS + 0, *reinterpret_cast<const uint32_t(*)[32]>(&pk[0]));
        // O correction (PV(j-1) has completed: S(j) was issued after it).
        if (j > 0 && __any_sync(0xffffffffu, alpha != 1.0f)) {
          const uint32_t tO = tmem + 256 + t * 128 + (static_cast<uint32_t>((warp & 3) * 32) << 16);
#pragma unroll
          for (int c = 0; c < 128; c += 32) {
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
        mbar_arrive(bar(L::bPFull + t));
      }
      if (!ok) break;
      sc += n;
      // row sums for the epilogue, once it has read the previous unit's
      if (uc > 0 && !warp_wait(bar(L::bRowFree + t), (uc - 1) & 1, abort_flag)) {
        ok = false;
        break;
      }
      s_rowl[t * 128 + row] = lr;
      mbar_arrive(bar(L::bFinal + t));
      if (!*abort_flag && q_row < p.N)
        p.lse[static_cast<size_t>(bh) * p.N + q_row] =
            l > 0.f ? (m * sl2 + lg2_approx(l)) * 0.69314718055994531f : -INFINITY;
    }
    if (!ok) fail(p.status, abort_flag, 5);
  } else if (warp < 12) {
    // ----------------------------------------------------------------- epilogue ----------
    setmaxnreg_dec<R::kEpilogue>();
    const int row = threadIdx.x - 256;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    int oc[2] = {0, 0};  // PV products of each tile in earlier units (phases of bODone)
    bool ok = true;
    for (int si = 0, uc = 0; ok; ++si, ++uc) {
      const int u = warp_next_unit(si);
      if (u == kGaveUp) { ok = false; break; }
      if (u < 0) break;
      const Unit U = unit_of(u);
      for (int t = 0; t < 2; ++t) {
        const int n = U.n_t[t];
        if (!warp_wait(bar(L::bFinal + t), uc & 1, abort_flag) ||
            (n > 0 && !warp_wait(bar(L::bODone + t), (oc[t] + n - 1) & 1, abort_flag))) {
          ok = false;
          break;
        }
        oc[t] += n;
        tc_fence_after();
        const float lr_row = s_rowl[t * 128 + row];
        mbar_arrive(bar(L::bRowFree + t));
        const float inv_l = lr_row > 0.f ? p.o_scale / lr_row : 0.f;
        const uint32_t tO = tmem + 256 + t * 128 + lane_off;
        uint8_t* stage = gbase + L::kO + t * L::kOTile;
        if (lane == 0) bulk_wait_group_read0();  // the previous unit's store has read it
        __syncwarp();
#pragma unroll
        for (int c = 0; c < 128; c += 32) {
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
            const int chunk = c / 8 + q;  // 0 .. 15
            *reinterpret_cast<uint4*>(stage + (chunk >> 3) * L::kOBoxBytes +
                                      sw128_offset(row, chunk & 7)) = v;
          }
        }
        tc_fence_before();
        mbar_arrive(bar(L::bOFree + t));  // O(t) is out of TMEM: the next unit may overwrite it
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          for (int b = 0; b < p.o_boxes; ++b)
            tma_store_3d(&tmO,
                         sbase + L::kO + t * L::kOTile + b * L::kOBoxBytes + (warp & 3) * 4096,
                         64 * b, U.q0 + t * 128 + (warp & 3) * 32, U.bh);
          bulk_commit_group();
        }
      }
    }
    if (!ok) fail(p.status, abort_flag, 5);
    if (lane == 0) bulk_wait_group0();
  } else {
    setmaxnreg_dec<R::kMma>();
    if (warp == 12 && lane == 0) {
      // ------------------------------------------------------------------ MMA -------------
      constexpr uint32_t idesc = idesc_e4m3_f32(128, 128);  // QK^T and PV: M = N = 128
      const uint64_t desc_q0 = sdesc_sw128(sbase + L::kQ, 16, 1024);
      const uint64_t desc_kv0 = sdesc_sw128(sbase + L::kKV, 16, 1024);
      // tt: the CTA's K/V load number (K of key tile j is load tb + 2j, V^T load tb + 2j + 1)
      auto wait_full = [&](int tt) -> bool {
        return mbar_wait(bar(L::bKvFull + tt % ST), (tt / ST) & 1, abort_flag);
      };
      auto issue_s = [&](int t, int tt) {
        const uint64_t a0 = sdesc_advance(desc_q0, t * L::kTile);
        const uint64_t b0 = sdesc_advance(desc_kv0, (tt % ST) * L::kTile);
        const uint32_t d = tmem + t * 128;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // 32 E4M3 (32 bytes) of the head dimension per step
          umma_ss_f8(d, sdesc_advance(a0, kk * 32), sdesc_advance(b0, kk * 32), idesc,
                     kk > 0 ? 1u : 0u);
        umma_commit(bar(L::bSFull + t));
      };
      auto issue_pv = [&](int t, int tt, bool acc) {
        const uint64_t b0 = sdesc_advance(desc_kv0, (tt % ST) * L::kTile);
        const uint32_t d = tmem + 256 + t * 128, a = tmem + t * 128;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // 32 keys per step: 8 TMEM columns of P
          umma_ts_f8(d, a + kk * 8, sdesc_advance(b0, kk * 32), idesc, (acc || kk > 0) ? 1u : 0u);
        umma_commit(bar(L::bODone + t));
      };
      bool ok = true;
      int tb = 0;
      int pc[2] = {0, 0};
      for (int si = 0, uc = 0; ok; ++si, ++uc) {
        if (!(ok = mbar_wait(bar(L::bSchedFull + (si & 1)), (si >> 1) & 1, abort_flag))) break;
        const int u = sched[si & 1];
        mbar_arrive(bar(L::bSchedEmpty + (si & 1)));
        if (u < 0) break;
        const Unit U = unit_of(u);
        const int n0 = U.n_t[0], n1 = U.n_t[1];
        if (!(ok = mbar_wait(bar(L::bQ), uc & 1, abort_flag) && (n1 == 0 || wait_full(tb)))) break;
        tc_fence_after();
        if (n1 > 0) {
          if (n0 > 0) issue_s(0, tb);
          issue_s(1, tb);
          umma_commit(bar(L::bKvEmpty + tb % ST));
        }
        if (n1 <= 1) umma_commit(bar(L::bQEmpty));  // no further S reads this unit's Q
        for (int j = 0; j < n1 && ok; ++j) {
          const int tv = tb + 2 * j + 1, tk = tb + 2 * j + 2;
          if (!wait_full(tv)) { ok = false; break; }
          tc_fence_after();
          if (j < n0) {
            if (!mbar_wait(bar(L::bPFull + 0), (pc[0] + j) & 1, abort_flag) ||
                (j == 0 && uc > 0 && !mbar_wait(bar(L::bOFree + 0), (uc - 1) & 1, abort_flag))) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_pv(0, tv, j > 0);
          }
          const bool more = j + 1 < n1;
          if (more) {
            if (!wait_full(tk)) { ok = false; break; }
            tc_fence_after();
            if (j + 1 < n0) issue_s(0, tk);
          }
          if (!mbar_wait(bar(L::bPFull + 1), (pc[1] + j) & 1, abort_flag) ||
              (j == 0 && uc > 0 && !mbar_wait(bar(L::bOFree + 1), (uc - 1) & 1, abort_flag))) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_pv(1, tv, j > 0);
          umma_commit(bar(L::bKvEmpty + tv % ST));
          if (more) {
            issue_s(1, tk);
            umma_commit(bar(L::bKvEmpty + tk % ST));
            if (j + 2 == n1) umma_commit(bar(L::bQEmpty));
          }
        }
        tb += 2 * n1;
        pc[0] += n0;
        pc[1] += n1;
      }
      if (!ok) fail(p.status, abort_flag, 5);
      // every MMA issued completes before TMEM is freed (bounded wait)
      volatile int never = 0;
      umma_commit(bar(L::bDrain));
      mbar_wait(bar(L::bDrain), 0, &never);
    } else if (warp == 13 && lane == 0) {
      // ------------------------------------------------- TMA, and the unit scheduler -------
      bool ok = true;
      int issued = 0, q_loads = 0, clc_n = 0;
      bool clc_pending = false;
      int u = static_cast<int>(blockIdx.x);
      for (int si = 0; ok; ++si) {
        if (!mbar_wait(bar(L::bSchedEmpty + (si & 1)), ((si >> 1) & 1) ^ 1, abort_flag)) {
          ok = false;
          break;
        }
        sched[si & 1] = u;
        mbar_arrive(bar(L::bSchedFull + (si & 1)));
        if (u < 0) break;
        const Unit U = unit_of(u);
        const int bh_kv = U.bh / p.group;
        if (si > 0 && !mbar_wait(bar(L::bQEmpty), (si - 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(bar(L::bQ), 2 * L::kTile);
#pragma unroll
        for (int t = 0; t < 2; ++t)
          tma_load_3d(sbase + L::kQ + t * L::kTile, &tmQ, bar(L::bQ), 0, U.q0 + 128 * t, U.bh);
        q_loads = si + 1;
        for (int j = 0; j < U.n_t[1] && ok; ++j) {
#pragma unroll
          for (int w = 0; w < 2; ++w) {
            const int tt = issued;
            const int st = tt % ST;
            if (!mbar_wait(bar(L::bKvEmpty + st), ((tt / ST) & 1) ^ 1, abort_flag)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(bar(L::bKvFull + st), L::kTile);
            const uint32_t dst = sbase + L::kKV + st * L::kTile;
            if (w == 0)
              tma_load_3d(dst, &tmK, bar(L::bKvFull + st), 0, 128 * j, bh_kv);  // K rows
            else
              tma_load_3d(dst, &tmVt, bar(L::bKvFull + st), 128 * j, 0, bh_kv);  // V^T rows
            issued = tt + 1;
          }
        }
        if (!ok) break;
        // claim the next unit once this one's loads are all issued
        mbar_arrive_expect_tx(bar(L::bClc), 16);
        clc_try_cancel(sbase + L::kClc, bar(L::bClc));
        clc_pending = true;
        ++clc_n;
        if (!mbar_wait(bar(L::bClc), (clc_n - 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        clc_pending = false;
        u = clc_cancelled_x(sbase + L::kClc);
      }
      if (!ok) fail(p.status, abort_flag, 5);
      // loads in flight and a pending launch-control reply land before the CTA exits
      volatile int never = 0;
#pragma unroll 1
      for (int tt = max(0, issued - ST); tt < issued; ++tt)
        mbar_wait(bar(L::bKvFull + tt % ST), (tt / ST) & 1, &never);
      if (q_loads > 0) mbar_wait(bar(L::bQ), (q_loads - 1) & 1, &never);
      if (clc_pending) mbar_wait(bar(L::bClc), (clc_n - 1) & 1, &never);
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

// V [rows][d] (E4M3 bytes) -> V^T [d][ld] per head. A block transposes 128 keys x 64 columns:
// each thread loads 4 x 4-byte blocks (four 32-bit words from rows r .. r+3), turns them into
// the four columns' words with byte permutes, and writes those to shared memory; the block then
// stores rows of 128 transposed keys with 16-byte stores. (Byte-wide shared-memory accesses,
// one per element, made an earlier version several times slower than a copy.)
// Grid: (ceil(N_kv / 128), ceil(d / 64), B * H_kv), 256 threads; d a multiple of 16.
constexpr int kTrKeys = 128;
__global__ void __launch_bounds__(256)
    fa_fp8_transpose_v(const uint8_t* __restrict__ v, uint8_t* __restrict__ vt, int N_kv, int d,
                       int ld) {
  // T[c][k / 4]: column c (0..63) of the tile, keys as bytes; rows of 128 keys padded to 144 bytes
  __shared__ __align__(16) uint32_t T[64][36];
  const int k0 = blockIdx.x * kTrKeys, c0 = blockIdx.y * 64;
  const size_t head = blockIdx.z;
#pragma unroll
  for (int rep = 0; rep < 2; ++rep) {
    // 4 x 4 block number (512 per tile): a warp covers 8 row groups x 4 column groups
    const int b = threadIdx.x + 256 * rep;
    const int rg = (b & 7) | (((b >> 5) & 3) << 3);  // 0 .. 31: keys 4 rg .. 4 rg + 3
    const int cg = ((b >> 3) & 3) | ((b >> 7) << 2);  // 0 .. 15: columns 4 cg .. 4 cg + 3
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      w[i] = 0u;
      if (k0 + 4 * rg + i < N_kv && c0 + 4 * cg < d)  // d % 16 == 0: the whole word is inside
        w[i] = *reinterpret_cast<const uint32_t*>(v + (head * N_kv + k0 + 4 * rg + i) * d + c0 +
                                                  4 * cg);
    }
    // byte j of word i is element (key 4 rg + i, column 4 cg + j); gather each column's bytes
    const uint32_t t0 = __byte_perm(w[0], w[1], 0x5140), t1 = __byte_perm(w[0], w[1], 0x7362);
    const uint32_t t2 = __byte_perm(w[2], w[3], 0x5140), t3 = __byte_perm(w[2], w[3], 0x7362);
    T[4 * cg + 0][rg] = __byte_perm(t0, t2, 0x5410);
    T[4 * cg + 1][rg] = __byte_perm(t0, t2, 0x7632);
    T[4 * cg + 2][rg] = __byte_perm(t1, t3, 0x5410);
    T[4 * cg + 3][rg] = __byte_perm(t1, t3, 0x7632);
  }
  __syncthreads();
#pragma unroll
  for (int rep = 0; rep < 2; ++rep) {
    const int e = threadIdx.x + 256 * rep;  // 16-byte chunk: 64 columns x 8 chunks of keys
    const int c = e >> 3, part = (e & 7) * 16;
    if (c0 + c < d && k0 + part < N_kv)  // ld % 16 == 0: the chunk fits in the row
      *reinterpret_cast<uint4*>(vt + (head * d + c0 + c) * static_cast<size_t>(ld) + k0 + part) =
          *reinterpret_cast<const uint4*>(&T[c][part / 4]);
  }
}

}  // namespace fa

// fa_fwd.cuh — exact attention forward for sm_100a (TMA + tcgen05 + TMEM, warp specialised).
//
// Computes, for every (batch, head) and query row i,
//     O_i = sum_j softmax_j(scale * q_i . k_j) v_j      and      lse_i = m_i + ln l_i,
// tile by tile with the online-softmax running max m and running sum l, so the N x N score
// and probability matrices never leave the SM ("How FlashAttention Actually Works: Tiling,
// SRAM Reuse, and Why It's 10x Faster", sections "How Tiling Works" and "The Secret Weapon:
// Online Softmax"; update rule of "How does FlashAttention optimize memory and speed via
// tiling?", "Core Technical Innovations" item 2).
//
// A work unit is two 128-row query tiles (256 rows) of one head; K/V stream through a
// shared-memory ring in 128-key tiles. The grid has one CTA per unit, but the kernel is
// persistent: each running CTA claims the next not-yet-launched CTA of the grid with cluster
// launch control and does its unit too, so units go out in launch order (grouped_unit's
// longest-first order) to whichever SM frees up, and one unit's epilogue and the next unit's
// Q and K/V loads overlap the current unit's last products. Roles (16 warps):
//   warps 0-3   softmax for query tile 0   (one thread per row, S read from TMEM)
//   warps 4-7   softmax for query tile 1
//   warps 8-11  epilogue (O / l -> bf16 -> TMA store)
//   warp 12     tcgen05.mma issue (one thread)
//   warp 13     TMA producer and unit scheduler (one thread)
//   warps 14-15 idle
// TMEM (512 columns): S0 [0,128), S1 [128,256), O0 [256,256+D), O1 [256+D,256+2D).
// P (bf16) is written back over the first 64 columns of its S buffer and fed to the PV MMA
// straight from TMEM, so P never touches shared memory.
// MMA issue order per key tile j: PV0(j), S0(j+1), PV1(j), S1(j+1) — while softmax 0 works on
// S0(j+1) the tensor core runs PV1(j) and S1(j+1), and vice versa.
// Variants: grouped K/V heads (query head h reads K/V head h / group), a causal offset for
// unequal lengths (key j visible to query i iff j <= i + off), and dropout on P (DROPOUT; keep
// decisions from dropout.cuh).
#pragma once
#include "dropout.cuh"
#include "sm100.cuh"

namespace fa {

constexpr int kFwdThreads = 512;
// Register split (setmaxnreg): softmax warps 0-7, epilogue warps 8-11, MMA/TMA warps 12-15.
// setmaxnreg.inc waits until the decrements have freed enough registers, so the split must add
// up to exactly the launch allocation (512 threads x 128 registers; checked on the host).
// The d = 64 dropout variant moves 16 registers per thread from the MMA/TMA warps (whose d = 64
// issue loop needs fewer) to the softmax warps, which also run the random-number generator.
template <int D, bool DROPOUT>
struct FwdRegs {
  static constexpr bool kShift = DROPOUT && D == 64;
  static constexpr uint32_t kSoftmax = kShift ? 184 : 176;
  static constexpr uint32_t kEpilogue = 64;
  static constexpr uint32_t kMma = kShift ? 80 : 96;
  static_assert(256 * kSoftmax + 128 * kEpilogue + 128 * kMma == kFwdThreads * 128,
                "forward register split must equal the launch allocation");
  // the softmax warps raise their count (setmaxnreg.inc), the others lower it (.dec)
  static_assert(kSoftmax > 128 && kEpilogue < 128 && kMma < 128, "setmaxnreg directions");
};
// Running-max update threshold, log2 units (exponentials stay below 2^8 between updates).
constexpr float kRescaleLog2 = 8.0f;

template <int D>
struct FwdLayout {
  static constexpr int kTileBytes = 128 * D * 2;  // one 128 x D bf16 tile
  static constexpr int kBoxBytes = 128 * 64 * 2;  // one TMA box: 128 rows x 64 columns
  static constexpr int kBoxes = D / 64;           // boxes per tile (128-byte swizzle rows)
  static constexpr int kStages = (D == 128) ? 4 : 8;
  static constexpr int kQ = 0;                                  // Q0, Q1
  static constexpr int kKV = 2 * kTileBytes;                    // K/V ring
  static constexpr int kOStage = kKV + kStages * kTileBytes;    // O staging: 4 warps x 4 KB
  static constexpr int kBars = kOStage + 4 * 4096;              // mbarriers
  static constexpr int kNumBars = 1 + 2 * kStages + 19;
  static constexpr int kRowL = kBars + kNumBars * 8;            // float[2][128]
  static constexpr int kSched = kRowL + 2 * 128 * 4;            // two unit indices
  static constexpr int kClc = (kSched + 8 + 15) / 16 * 16;      // 16-byte launch-control reply
  static constexpr int kTmemSlot = kClc + 16;
  static constexpr int kBytes = kTmemSlot + 16;
  static constexpr int kAlloc = kBytes + 1024;  // slack for 1024-byte alignment of the base

  // barrier indices
  static constexpr int bQ = 0;                       // Q0 and Q1 of the unit
  static constexpr int bKvFull = 1;                  // + stage
  static constexpr int bKvEmpty = 1 + kStages;       // + stage
  static constexpr int bSFull = 1 + 2 * kStages;     // + tile
  static constexpr int bPFull = bSFull + 2;          // + tile (128 arrivals)
  static constexpr int bODone = bSFull + 4;          // + tile
  static constexpr int bFinal = bSFull + 6;          // + tile (128 arrivals): row sums written
  static constexpr int bOFree = bSFull + 8;          // + tile (128): O read out of TMEM
  static constexpr int bRowFree = bSFull + 10;       // + tile (128): row sums read
  static constexpr int bSchedFull = bSFull + 12;     // + slot: next unit published
  static constexpr int bSchedEmpty = bSFull + 14;    // + slot: read by every consuming warp
  static constexpr int bQEmpty = bSFull + 16;        // every S of the unit completed
  static constexpr int bClc = bSFull + 17;           // launch-control reply landed
  static constexpr int bDrain = bSFull + 18;         // error path only
  static constexpr int kSchedReaders = 13;           // warps 0-11 and the MMA thread
};

struct FwdParams {
  float* lse;       // [BH, N] fp32
  int* status;      // device status word (FA_ERR_TIMEOUT on a timed-out wait)
  int N;            // query rows per head
  int N_kv;         // key/value rows per head
  int BH;           // batch * query heads
  int group;        // query heads per key/value head (1 unless K/V heads are shared)
  int off;          // causal offset: key j visible to query i iff j <= i + off
  int n_qblocks;    // query blocks per head
  int hgroup;       // query heads per scheduling group (see fwd_work_unit)
  float scale;      // softmax scale
  float scale_log2; // scale * log2(e)
  DropoutParams drop;  // read only by the DROPOUT instantiations
  // Failure-detection test hook (off by default): the producer never issues K/V load number
  // dbg_skip of each CTA, so the MMA warp's wait for it runs out after limit_ns and the kernel
  // unwinds with FA_ERR_TIMEOUT. limit_ns bounds the MMA warp's waits.
  int dbg_skip = -1;
  unsigned long long limit_ns = FA_SPIN_LIMIT_NS;
};

// Work unit `b` of a grid covering n_heads heads x n_tiles tiles, heads taken in groups of
// `group` (sized on the host so that a group's shared operands stay in L2 while its units run;
// the hardware hands out blocks roughly in index order, so a group's units run together). Inside
// a group, tile rank 0 (the heaviest tile) comes first for every head of the group, then rank 1,
// and so on (longest-processing-time order). When `group` does not divide n_heads, the smaller
// group goes first: run last, its heaviest units would start when every other unit has been
// handed out and end well after them.
__device__ __forceinline__ void grouped_unit(int b, int n_tiles, int n_heads, int group, int& rank,
                                             int& head) {
  const int rem = n_heads % group;
  const int first = rem * n_tiles;  // units of the smaller group
  int g0, gcur, r;
  if (b < first) {
    g0 = n_heads - rem;
    gcur = rem;
    r = b;
  } else {
    b -= first;
    g0 = (b / (group * n_tiles)) * group;
    gcur = group;
    r = b % (group * n_tiles);
  }
  rank = r / gcur;
  head = g0 + r % gcur;
}

// Work unit of CTA `cta` in a forward grid of n_qblocks * BH CTAs: query block qb of query head
// bh, in groups of `hgroup` query heads whose K and V stay in L2; causal work grows with the
// query block index, so the last blocks are the heaviest.
__device__ __forceinline__ void fwd_work_unit(int cta, int n_qblocks, int BH, int hgroup, int& qb,
                                              int& bh) {
  int rank;
  grouped_unit(cta, n_qblocks, BH, hgroup, rank, bh);
  qb = n_qblocks - 1 - rank;
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float lg2_approx(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <uint32_t R>
__device__ __forceinline__ void setmaxnreg_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(R));
}
template <uint32_t R>
__device__ __forceinline__ void setmaxnreg_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(R));
}

// Bounded wait whose result is the same on every lane of the warp (needed before the
// warp-collective tcgen05.ld / tcgen05.st that follow it).
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort));
}

__device__ __forceinline__ void fail(int* status, volatile int* abort_flag, int code) {
  *abort_flag = 1;
  atomicExch(status, code);
}

// D: the shared-memory and TMEM layout (64 or 128 columns of d). DM: the head dimension the
// products run over (D, or 96 with the d = 128 layout; the tensor maps zero-fill columns past d,
// so a 96-column contraction over them is exact).
template <int D, bool CAUSAL, bool DROPOUT, int DM = D>
__global__ void __launch_bounds__(kFwdThreads, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                  const FwdParams p) {
  using L = FwdLayout<D>;
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
  // Unit u: query block qb (rows [256 qb, 256 qb + 256)) of query head bh; key tiles each of its
  // two query tiles visits: all of them, or (causal) up to the one holding the last key its last
  // row sees; 0 when no row of the tile sees any key.
  struct Unit {
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
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmO);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(gbase + L::kTmemSlot);

  // Unit number s of this CTA, as a whole warp: wait for the producer to publish it, then
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
    // ------------------------------------------------------------------ softmax ----------
    setmaxnreg_inc<FwdRegs<D, DROPOUT>::kSoftmax>();
    const int t = warp >> 2;
    const int row = threadIdx.x & 127;
    const uint32_t tS = tmem + t * 128 + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const float sl2 = p.scale_log2;
    int sc = 0;  // S tiles of this query tile in earlier units (phases of bSFull, bPFull)
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
      float lr = 0.f;  // sum of the same exponentials rounded to bf16: normalises O, whose
                       // PV MMA used exactly those rounded weights
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
          const int lim = CAUSAL ? min(q_row + 1 + p.off, p.N_kv) : p.N_kv;  // keys [0, lim)
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
        // The running max is raised only when a tile's max exceeds it by more than
        // kRescaleLog2 (in log2 units): until then exponentials stay below 2^kRescaleLog2, and
        // the final O / l and lse = m + ln l use the same (stale) m, so the result is exact.
        const float m_tile = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3));
        float alpha = 1.0f;
        if ((m_tile - m) * sl2 > kRescaleLog2) {  // always true on the first tile (m = -inf)
          alpha = ex2_approx((m - m_tile) * sl2);  // 0 on the first tile
          m = m_tile;
        }
        // a row that has seen no key yet keeps m = -inf; its exponentials are then exactly 0
        const float nb = m == -INFINITY ? 0.f : -m * sl2;
        const uint64_t sl2x2 = f2_pack(sl2, sl2), nbx2 = f2_pack(nb, nb);
        uint64_t lsum[4] = {0, 0, 0, 0}, rsum[4] = {0, 0, 0, 0};  // (0.f, 0.f) pairs
        uint32_t pk[64];
        if constexpr (!DROPOUT) {
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
        } else {
          // Dropout: the sums l, lr take every weight; the P handed to the PV MMA keeps only the
          // kept ones (the keep scale is applied with 1/lr in the epilogue). Keys are taken 16
          // at a time: the quad's four lanes each run one generator call (one 4 x 4 block) and
          // swap words so that each lane holds its own row's bytes for the 16 keys.
#pragma unroll
          for (int mc = 0; mc < 8; ++mc) {
            uint32_t kw[4] = {static_cast<uint32_t>(32 * j + 4 * mc + (lane & 3)),
                              static_cast<uint32_t>(q_row) >> 2, static_cast<uint32_t>(bh),
                              p.drop.offset};
            philox4x32_10(kw, p.drop.seed_lo, p.drop.seed_hi);
            quad_transpose(kw, lane);  // kw[g]: bytes of keys 16 mc + 4 g + (0..3), this row
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              const uint32_t kb = keep_bytes(kw[g], p.drop.add4);
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const int c = 16 * mc + 4 * g + 2 * h;
                float a0, a1;
                f2_unpack(f2_fma(f2_pack_u(s[c], s[c + 1]), sl2x2, nbx2), a0, a1);
                const float e0 = ex2_approx(a0), e1 = ex2_approx(a1);
                const uint32_t w = pack_bf16x2(e0, e1);
                pk[c / 2] = w & (h == 0 ? pair_mask<0>(kb) : pair_mask<1>(kb));
                lsum[(c >> 1) & 3] = f2_add(lsum[(c >> 1) & 3], f2_pack(e0, e1));
                rsum[(c >> 1) & 3] = f2_add(rsum[(c >> 1) & 3], f2_pack_u(w << 16, w & 0xffff0000u));
              }
            }
          }
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
        // O correction. S(j) was issued after PV(j-1) and tcgen05 MMAs complete in order, so
        // PV(j-1) has finished: O can be rescaled here without another wait. PV(j) is issued
        // only after the arrive below.
        if (j > 0 && __any_sync(0xffffffffu, alpha != 1.0f)) {
          const uint32_t tO = tmem + 256 + t * D + (static_cast<uint32_t>((warp & 3) * 32) << 16);
#pragma unroll
          for (int c = 0; c < DM; c += 32) {
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
      // rows that saw no key: O = 0 and lse = -inf
      if (!*abort_flag && q_row < p.N)
        p.lse[static_cast<size_t>(bh) * p.N + q_row] =
            l > 0.f ? (m * sl2 + lg2_approx(l)) * 0.69314718055994531f : -INFINITY;
    }
    if (!ok) fail(p.status, abort_flag, 5);
  } else if (warp < 12) {
    // ----------------------------------------------------------------- epilogue ----------
    setmaxnreg_dec<FwdRegs<D, DROPOUT>::kEpilogue>();
    const int w4 = warp & 3;                       // rows [32 w4, 32 w4 + 32) of each tile
    const int row = threadIdx.x - 256;
    const uint32_t lane_off = static_cast<uint32_t>(w4 * 32) << 16;
    uint8_t* stage = gbase + L::kOStage + w4 * 4096;
    const uint32_t stage_s = sbase + L::kOStage + w4 * 4096;
    int oc[2] = {0, 0};  // PV products of each tile in earlier units (phases of bODone)
    bool ok = true;
    // O = O_acc / l  ->  bf16  ->  this warp's 4 KB staging box (32 rows x 64 columns,
    // 128-byte swizzle)  ->  TMA store, one 64-column box at a time. Each warp stores its own
    // rows, so no cross-warp barrier is needed.
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
        float inv_l = lr_row > 0.f ? 1.0f / lr_row : 0.f;
        if constexpr (DROPOUT) inv_l = lr_row > 0.f ? p.drop.keep_scale / lr_row : 0.f;
        const uint32_t tO = tmem + 256 + t * D + lane_off;
#pragma unroll
        for (int b = 0; b < L::kBoxes; ++b) {
          if (lane == 0) bulk_wait_group_read0();  // the previous store has read the staging
          __syncwarp();
#pragma unroll
          for (int c = 64 * b; c < 64 * b + 64; c += 32) {
            uint32_t o[32];
            if (n > 0 && c < DM) {
              tmem_ld_32x32b_x32(tO + c, o);
              tmem_ld_wait();
              reg_fence(o);
            } else {  // no PV ever wrote these O columns (past d, which the store clips)
#pragma unroll
              for (int i = 0; i < 32; ++i) o[i] = 0u;
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {  // four 16-byte chunks of 8 columns
              uint4 v;
              v.x = pack_bf16x2(__uint_as_float(o[8 * q + 0]) * inv_l, __uint_as_float(o[8 * q + 1]) * inv_l);
              v.y = pack_bf16x2(__uint_as_float(o[8 * q + 2]) * inv_l, __uint_as_float(o[8 * q + 3]) * inv_l);
              v.z = pack_bf16x2(__uint_as_float(o[8 * q + 4]) * inv_l, __uint_as_float(o[8 * q + 5]) * inv_l);
              v.w = pack_bf16x2(__uint_as_float(o[8 * q + 6]) * inv_l, __uint_as_float(o[8 * q + 7]) * inv_l);
              *reinterpret_cast<uint4*>(stage + sw128_offset(lane, ((c & 63) >> 3) + q)) = v;
            }
          }
          if (b == L::kBoxes - 1) {  // all of O(t) is out of TMEM: the next unit may overwrite it
            tc_fence_before();
            mbar_arrive(bar(L::bOFree + t));
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_3d(&tmO, stage_s, 64 * b, U.q0 + t * 128 + w4 * 32, U.bh);
            bulk_commit_group();
          }
        }
      }
    }
    if (!ok) fail(p.status, abort_flag, 5);
    if (lane == 0) bulk_wait_group0();
  } else {
    setmaxnreg_dec<FwdRegs<D, DROPOUT>::kMma>();
    if (warp == 12 && lane == 0) {
      // ------------------------------------------------------------------ MMA -------------
      const uint32_t idesc_qk = idesc_bf16_f32(128, 128, false, false);
      const uint32_t idesc_pv = idesc_bf16_f32(128, DM, false, true);
      // Operand descriptors are built once; per k-step they are advanced by constant offsets.
      const uint64_t desc_q0 = sdesc_sw128(sbase + L::kQ, 16, 1024);             // K-major
      const uint64_t desc_k0 = sdesc_sw128(sbase + L::kKV, 16, 1024);            // K-major
      const uint64_t desc_v0 = sdesc_sw128(sbase + L::kKV, L::kBoxBytes, 1024);  // MN-major
      // tt: the CTA's K/V load number (K of key tile j is load tb + 2j, V load tb + 2j + 1)
      auto wait_full = [&](int tt) -> bool {
        return mbar_wait(bar(L::bKvFull + tt % ST), (tt / ST) & 1, abort_flag, p.limit_ns);
      };
      auto issue_s = [&](int t, int tt) {
        const uint64_t a0 = sdesc_advance(desc_q0, t * L::kTileBytes);
        const uint64_t b0 = sdesc_advance(desc_k0, (tt % ST) * L::kTileBytes);
        const uint32_t d = tmem + t * 128;
#pragma unroll
        for (int kk = 0; kk < DM / 16; ++kk) {
          const uint32_t off = (kk >> 2) * L::kBoxBytes + (kk & 3) * 32;
          umma_ss(d, sdesc_advance(a0, off), sdesc_advance(b0, off), idesc_qk, kk > 0 ? 1u : 0u);
        }
        umma_commit(bar(L::bSFull + t));
      };
      auto issue_pv = [&](int t, int tt, bool acc) {
        const uint64_t b0 = sdesc_advance(desc_v0, (tt % ST) * L::kTileBytes);
        const uint32_t d = tmem + 256 + t * D, a = tmem + t * 128;
        umma_ts(d, a, b0, idesc_pv, acc ? 1u : 0u);
#pragma unroll
        for (int kk = 1; kk < 8; ++kk)
          umma_ts(d, a + kk * 8, sdesc_advance(b0, kk * 2048), idesc_pv, 1u);
        umma_commit(bar(L::bODone + t));
      };
      const uint64_t lim = p.limit_ns;
      bool ok = true;
      int tb = 0;            // K/V loads of earlier units
      int pc[2] = {0, 0};    // P tiles of earlier units (phases of bPFull)
      for (int si = 0, uc = 0; ok; ++si, ++uc) {
        if (!(ok = mbar_wait(bar(L::bSchedFull + (si & 1)), (si >> 1) & 1, abort_flag, lim))) break;
        const int u = sched[si & 1];
        mbar_arrive(bar(L::bSchedEmpty + (si & 1)));
        if (u < 0) break;
        const Unit U = unit_of(u);
        const int n0 = U.n_t[0], n1 = U.n_t[1];
        // the unit's Q (and its first K, when it has one)
        if (!(ok = mbar_wait(bar(L::bQ), uc & 1, abort_flag, lim) && (n1 == 0 || wait_full(tb))))
          break;
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
            // the unit's first PV(0) overwrites O(0), which the epilogue of the previous unit
            // reads out of TMEM first
            if (!mbar_wait(bar(L::bPFull + 0), (pc[0] + j) & 1, abort_flag, lim) ||
                (j == 0 && uc > 0 && !mbar_wait(bar(L::bOFree + 0), (uc - 1) & 1, abort_flag, lim))) {
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
          if (!mbar_wait(bar(L::bPFull + 1), (pc[1] + j) & 1, abort_flag, lim) ||
              (j == 0 && uc > 0 && !mbar_wait(bar(L::bOFree + 1), (uc - 1) & 1, abort_flag, lim))) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_pv(1, tv, j > 0);
          umma_commit(bar(L::bKvEmpty + tv % ST));
          if (more) {
            issue_s(1, tk);
            umma_commit(bar(L::bKvEmpty + tk % ST));
            if (j + 2 == n1) umma_commit(bar(L::bQEmpty));  // that was the unit's last S
          }
        }
        tb += 2 * n1;
        pc[0] += n0;
        pc[1] += n1;
      }
      if (!ok) fail(p.status, abort_flag, 5);
      // Every MMA this thread issued completes before tensor memory is freed and the CTA exits
      // (on the normal path the epilogue waits for the same products; after a give-up this is
      // the drain). Bounded wait.
      volatile int never = 0;
      umma_commit(bar(L::bDrain));
      mbar_wait(bar(L::bDrain), 0, &never);
    } else if (warp == 13 && lane == 0) {
      // ------------------------------------------------- TMA, and the unit scheduler -------
      bool ok = true;
      int issued = 0;        // K/V loads issued (the CTA's load numbers run across units)
      int q_loads = 0;       // units whose Q load was issued
      bool clc_pending = false;
      int clc_n = 0;         // launch-control requests issued
      int u = static_cast<int>(blockIdx.x);
      for (int si = 0; ok; ++si) {
        // publish unit si of this CTA (-1 when none is left) once every reader took unit si-2
        if (!mbar_wait(bar(L::bSchedEmpty + (si & 1)), ((si >> 1) & 1) ^ 1, abort_flag)) {
          ok = false;
          break;
        }
        sched[si & 1] = u;
        mbar_arrive(bar(L::bSchedFull + (si & 1)));
        if (u < 0) break;
        const Unit U = unit_of(u);
        const int bh_kv = U.bh / p.group;  // key/value head of this query head
        // Q of the unit, once every S of the previous unit has completed
        if (si > 0 && !mbar_wait(bar(L::bQEmpty), (si - 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(bar(L::bQ), 2 * L::kTileBytes);
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
          for (int b = 0; b < L::kBoxes; ++b)
            tma_load_3d(sbase + L::kQ + t * L::kTileBytes + b * L::kBoxBytes, &tmQ, bar(L::bQ),
                        64 * b, U.q0 + 128 * t, U.bh);
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
            if (tt != p.dbg_skip) {  // (the test hook leaves this load out)
              mbar_arrive_expect_tx(bar(L::bKvFull + st), L::kTileBytes);
              const uint32_t dst = sbase + L::kKV + st * L::kTileBytes;
#pragma unroll
              for (int b = 0; b < L::kBoxes; ++b)
                tma_load_3d(dst + b * L::kBoxBytes, w ? &tmV : &tmK, bar(L::bKvFull + st), 64 * b,
                            128 * j, bh_kv);
            }
            issued = tt + 1;
          }
        }
        if (!ok) break;
        // claim the next unit once this one's loads are all issued (as late as the prefetch
        // allows, so that a unit still unclaimed goes to whichever SM frees up first)
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
      // Every load issued (and a pending launch-control reply) lands before the CTA can exit,
      // whether or not (or whenever) a role gives up. The last ST loads are the latest in their
      // stages, so on the normal path these bounded waits return at once.
      volatile int never = 0;
#pragma unroll 1
      for (int tt = max(0, issued - ST); tt < issued; ++tt)
        if (tt != p.dbg_skip) mbar_wait(bar(L::bKvFull + tt % ST), (tt / ST) & 1, &never);
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

}  // namespace fa

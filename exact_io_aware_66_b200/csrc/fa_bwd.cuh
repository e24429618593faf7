// fa_bwd.cuh — exact attention backward for sm_100a.
//
// The backward stores nothing of size N x N: it recomputes the scores and probabilities on chip
// from Q, K and the forward's per-row logsumexp ("How FlashAttention Actually Works",
// section "The Backward Pass: Recomputation"; "Breaking the Memory Wall", section "Backward
// Pass Recomputation": only the normalisation factors are kept). With P = exp(S - lse):
//     dV = P^T dO,  dP = dO V^T,  D_i = dO_i . O_i,  dS = P o (dP - D),
//     dQ = scale dS K,  dK = scale dS^T Q
// (the calculus of softmax attention; the pages give no backward formulas).
//
// Three kernels run in order on the caller's stream:
//   1. fa_bwd_preprocess: D = rowsum(dO o O) (fp32), lse2 = -lse * log2(e), dQ_acc = 0.
//   2. fa_bwd_main: a persistent kernel whose work units are (key/value head, 128-key tile j),
//      each looping over every query head that shares the key/value head and over the 64-row
//      query tiles that see tile j (one CTA per SM takes units from a counter).
//      K_j and V_j stay in shared memory; tiles of Q and dO stream through a 3-stage TMA ring
//      (4 at d = 64). Per query tile i, five tcgen05 MMAs (all M = 128):
//          S^T  = K_j Q_i^T          -> TMEM (64 columns, double buffered)
//          dP^T = V_j dO_i^T         -> TMEM (64 columns, double buffered)
//          dV  += P^T dO_i           (A = P^T from TMEM, bf16)            -> TMEM, d columns
//          dK  += dS^T Q_i           (A = dS^T from shared memory)       -> TMEM, d columns
//          dQ^T = K_j^T dS^T         (both operands MN-major in shared memory) -> the dP^T buffer
//      Two warpgroups turn S^T/dP^T into P^T (back to TMEM) and dS^T (to shared memory) while
//      the tensor core works on the previous tile; a third drains dQ^T from TMEM and adds it
//      into the fp32 accumulator with TMA bulk reductions (cp.reduce.async.bulk .add.f32).
//      The final dK (times scale) and dV are stored with TMA by the drain warps, while the
//      others start the next unit. With dropout (DROPOUT), the
//      elementwise warps regenerate the keep decisions of the forward (dropout.cuh) and form
//      dS = P o (r Z o dP - D) and Z o P for the dV product; dV is scaled by r at the end.
//   3. fa_bwd_dq_convert: dQ = bf16(dQ_acc).
#pragma once
#include "dropout.cuh"
#include "fa_fwd.cuh"
#include "sm100.cuh"

namespace fa {

// Workspace layout (each section 256-byte aligned):
//   dQ_acc [BH, N, d] fp32 | D [BH, N64] fp32 | lse2 [BH, N64] fp32 | unit counter (int)
// where N64 = N rounded up to a multiple of 64, so every row of D and lse2 starts on a
// 256-byte boundary (TMA needs 16-byte aligned row strides). The counter hands out work units
// to the persistent 128-row backward kernel; the preprocess kernel zeroes it.
__host__ __device__ inline size_t bwd_align256(size_t x) { return (x + 255) / 256 * 256; }
inline size_t bwd_n64(int N) { return (static_cast<size_t>(N) + 63) / 64 * 64; }
inline size_t bwd_ws_offset_D(size_t BH, int N, int d) {
  return bwd_align256(BH * N * static_cast<size_t>(d) * 4);
}
inline size_t bwd_ws_offset_lse2(size_t BH, int N, int d) {
  return bwd_ws_offset_D(BH, N, d) + bwd_align256(BH * bwd_n64(N) * 4);
}
inline size_t bwd_ws_offset_sched(size_t BH, int N, int d) {
  return bwd_ws_offset_lse2(BH, N, d) + bwd_align256(BH * bwd_n64(N) * 4);
}
inline size_t bwd_workspace_bytes(size_t BH, int N, int d) {
  return bwd_ws_offset_sched(BH, N, d) + 256;
}

// ------------------------------------------------------------------------------------------
// 1. Preprocess: one group of TPR threads per row (d/8 rounded up to a power of two); each
//    thread owns 8 columns (threads past the row's d/8 chunks only join the reduction).
// ------------------------------------------------------------------------------------------
constexpr int kPrepThreads = 256;

template <int D>
__global__ void __launch_bounds__(kPrepThreads)
    fa_bwd_preprocess(const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ dO,
                      const float* __restrict__ lse, float* __restrict__ dq_acc,
                      float* __restrict__ Dvec, float* __restrict__ lse2, long long rows, int N,
                      int n64, int* __restrict__ counter) {
  constexpr int TPR = D <= 64 ? 8 : (D <= 128 ? 16 : 32);  // threads per row
  static_assert(D % 8 == 0 && D / 8 <= TPR, "preprocess row split");
  const long long t = static_cast<long long>(blockIdx.x) * kPrepThreads + threadIdx.x;
  const long long row = t / TPR;
  const int part = static_cast<int>(t % TPR);
  if (t == 0 && counter != nullptr) *counter = 0;  // unit counter of the persistent main kernel
  float acc = 0.f;
  if (row < rows && part * 8 < D) {
    const uint4 a = *reinterpret_cast<const uint4*>(o + row * D + part * 8);
    const uint4 b = *reinterpret_cast<const uint4*>(dO + row * D + part * 8);
    const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
    const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 fa2 = __bfloat1622float2(a2[i]);
      const float2 fb2 = __bfloat1622float2(b2[i]);
      acc = fmaf(fa2.x, fb2.x, acc);
      acc = fmaf(fa2.y, fb2.y, acc);
    }
    float4* z = reinterpret_cast<float4*>(dq_acc + row * D + part * 8);
    z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int off = TPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (row < rows && part == 0) {
    const long long padded = (row / N) * n64 + row % N;
    Dvec[padded] = acc;
    lse2[padded] = -lse[row] * 1.4426950408889634f;  // stored negated: P = 2^(S log2e scale + this)
  }
}

// ------------------------------------------------------------------------------------------
// 3. dQ conversion: fp32 accumulator (already scaled) -> bf16, 8 elements per thread.
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
    fa_bwd_dq_convert(const float* __restrict__ dq_acc, __nv_bfloat16* __restrict__ dq,
                      long long n8) {
  const long long t = static_cast<long long>(blockIdx.x) * 256 + threadIdx.x;
  if (t >= n8) return;
  const float4 a = reinterpret_cast<const float4*>(dq_acc)[2 * t];
  const float4 b = reinterpret_cast<const float4*>(dq_acc)[2 * t + 1];
  uint4 r;
  r.x = pack_bf16x2(a.x, a.y);
  r.y = pack_bf16x2(a.z, a.w);
  r.z = pack_bf16x2(b.x, b.y);
  r.w = pack_bf16x2(b.z, b.w);
  reinterpret_cast<uint4*>(dq)[t] = r;
}

// ------------------------------------------------------------------------------------------
// 2. Main kernel.
// ------------------------------------------------------------------------------------------
constexpr int kBwdThreads = 512;

template <int D>
struct BwdLayout {
  static constexpr int kKVBox = 128 * 64 * 2;   // K/V TMA box: 128 rows x 64 columns
  static constexpr int kQBox = 64 * 64 * 2;     // Q/dO TMA box: 64 rows x 64 columns
  static constexpr int kBoxes = D / 64;
  static constexpr int kKVTile = 128 * D * 2;
  static constexpr int kQTile = 64 * D * 2;
  static constexpr int kQStages = (D == 128) ? 3 : 4;  // Q/dO ring depth
  static constexpr int kK = 0;
  static constexpr int kV = kK + kKVTile;
  static constexpr int kQ = kV + kKVTile;               // + stage * 2 * kQTile
  static constexpr int kDO = kQ + kQTile;               // + stage * 2 * kQTile
  static constexpr int kDS = kQ + kQStages * 2 * kQTile;  // 2 x 16 KB: dS^T [128 keys][64 q]
  static constexpr int kDQ = kDS + 2 * 16384;           // 4 warps x 8 KB fp32 staging
  static constexpr int kRow = kDQ + 4 * 8192;           // per stage: lse2[64], D[64]
  static constexpr int kBars = kRow + kQStages * 512;

  static constexpr int bKV = 0;
  static constexpr int bQFull = 1;                      // + stage
  static constexpr int bQEmpty = 1 + kQStages;          // + stage
  static constexpr int bSdPFull = 1 + 2 * kQStages;     // + buffer
  static constexpr int bEwDone = bSdPFull + 2;          // + buffer (256 arrivals)
  static constexpr int bDQFull = bSdPFull + 4;          // + buffer
  static constexpr int bDQFree = bSdPFull + 6;          // + buffer (128 arrivals)
  static constexpr int bDSFree = bSdPFull + 8;          // + buffer
  static constexpr int bAccDone = bSdPFull + 10;
  static constexpr int bDrain = bSdPFull + 11;
  static constexpr int bAccFree = bSdPFull + 12;        // dV, dK of the unit read out (128)
  static constexpr int bSchedFull = bSdPFull + 13;      // + slot: next unit index published
  static constexpr int bSchedEmpty = bSdPFull + 15;     // + slot: read by every consuming warp
  static constexpr int kNumBars = bSdPFull + 17;
  static constexpr int kSchedReaders = 13;              // warps 0-11 and the MMA thread

  static constexpr int kSched = kBars + kNumBars * 8;  // two unit indices (-1: no unit left)
  static constexpr int kTmemSlot = kSched + 8;
  static constexpr int kBytes = kTmemSlot + 16;
  static constexpr int kAlloc = kBytes + 1024;

  // TMEM columns
  static constexpr uint32_t tDV = 0;
  static constexpr uint32_t tDK = D;
  __host__ __device__ static constexpr uint32_t tS(int b) { return 256u + 128u * b; }
  __host__ __device__ static constexpr uint32_t tDP(int b) { return 256u + 128u * b + 64u; }
};
// (plus the kernel's few bytes of static shared memory)
static_assert(BwdLayout<128>::kAlloc + 16 <= 227 * 1024, "64-row backward shared memory");

struct BwdParams {
  int* status;
  int N;           // query rows per head
  int N_kv;        // key/value rows per head
  int BH_kv;       // batch * key/value heads (one CTA row of the grid per key/value head)
  int qgroup;      // query heads per key/value head
  int off;         // causal offset: key j visible to query i iff j <= i + off
  int n_kv;        // ceil(N_kv / 128)
  int n_q;         // ceil(N / 64)
  int group;       // key/value heads per scheduling group
  int d;           // head dimension of the tensors (<= D; columns past d are zero-filled)
  float scale;
  float scale_log2;
  DropoutParams drop;  // read only by the DROPOUT instantiations
  // Failure-detection test hook (off by default): the producer never issues the Q tile of
  // iteration dbg_skip of each CTA, so the MMA warp's wait for it runs out after limit_ns and
  // the kernel unwinds with FA_ERR_TIMEOUT. limit_ns bounds the MMA warp's waits.
  int dbg_skip = -1;
  unsigned long long limit_ns = FA_SPIN_LIMIT_NS;
  // Persistent kernels (fa_bwd_q128.cuh): units n_kv * BH_kv in all, the first gridDim.x taken
  // by block index, the rest handed out by this zeroed counter.
  int n_units = 0;
  int* sched_counter = nullptr;
};

template <int D, bool CAUSAL, bool DROPOUT>
__global__ void __launch_bounds__(kBwdThreads, 1)
    fa_bwd_main(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                const __grid_constant__ CUtensorMap tmLse2, const __grid_constant__ CUtensorMap tmD,
                const __grid_constant__ CUtensorMap tmDQacc,
                const __grid_constant__ CUtensorMap tmDK, const __grid_constant__ CUtensorMap tmDV,
                const BwdParams p) {
  using L = BwdLayout<D>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ int abort_flag_storage;
  volatile int* abort_flag = &abort_flag_storage;

  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (sbase - raw);
  auto bar = [&](int i) -> uint32_t { return sbase + L::kBars + 8u * i; };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  constexpr int QS = L::kQStages;
  // The kernel is persistent: one CTA per SM (at most one per unit) takes work units — one
  // (key/value head, 128-key tile j) each — unit blockIdx.x first, then gridDim.x + the value
  // of a counter in the workspace (zeroed by the preprocess kernel), in the order of
  // grouped_unit: groups of p.group heads sized so that a group's Q, dO, K, V and dQ
  // accumulator fit in L2, the key tiles with the most query tiles first inside a group. A
  // unit loops over every query head that shares its key/value head and over the 64-row query
  // tiles that see its keys. Every pipeline barrier counts its phases over the CTA's run.
  struct Unit {
    int bh, k0, qi0, n_qt, n_i;
  };
  auto unit_of = [&](int u) {
    Unit w;
    int j;
    grouped_unit(u, p.n_kv, p.BH_kv, p.group, j, w.bh);
    w.k0 = 128 * j;
    // first 64-row query tile with a query that sees a key of this tile (j <= i + off)
    w.qi0 = CAUSAL ? max(0, w.k0 - p.off) / 64 : 0;
    w.n_qt = max(0, p.n_q - w.qi0);
    w.n_i = p.qgroup * w.n_qt;
    return w;
  };
  volatile int* sched = reinterpret_cast<volatile int*>(gbase + L::kSched);

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(bar(L::bKV), 1);
    for (int s = 0; s < QS; ++s) {
      mbar_init(bar(L::bQFull + s), 1);
      mbar_init(bar(L::bQEmpty + s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(L::bSdPFull + s), 1);
      mbar_init(bar(L::bEwDone + s), 256);
      mbar_init(bar(L::bDQFull + s), 1);
      mbar_init(bar(L::bDQFree + s), 128);
      mbar_init(bar(L::bDSFree + s), 1);
      mbar_init(bar(L::bSchedFull + s), 1);
      mbar_init(bar(L::bSchedEmpty + s), L::kSchedReaders);
    }
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
    // ------------------------------------------------------- P^T and dS^T (elementwise) ---
    const int w = warp >> 2;                       // query columns [32w, 32w+32)
    const int r = threadIdx.x & 127;               // key row within the tile (TMEM lane)
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const float sl2 = p.scale_log2;
    bool ok = true;
    int g = 0;  // tiles of this CTA's earlier units
    for (int si = 0; ok; ++si) {
      const int u = warp_next_unit(si);
      if (u == kGaveUp) { ok = false; break; }
      if (u < 0) break;
      const Unit U = unit_of(u);
      const int key = U.k0 + r;
      for (int i = 0; i < U.n_i && ok; ++i, ++g) {
        const int b = g & 1, st = g % QS;
        const int qi = U.qi0 + i % U.n_qt, qh = U.bh * p.qgroup + i / U.n_qt;
        ok = warp_wait(bar(L::bQFull + st), (g / QS) & 1, abort_flag) &&
             warp_wait(bar(L::bSdPFull + b), (g >> 1) & 1, abort_flag) &&
             (g < 2 || warp_wait(bar(L::bDSFree + b), ((g >> 1) & 1) ^ 1, abort_flag));
        if (!ok) break;
        tc_fence_after();
        uint32_t s[32], dp[32];
        tmem_ld_32x32b_x32(tmem + L::tS(b) + 32 * w + lane_off, s);
        tmem_ld_32x32b_x32(tmem + L::tDP(b) + 32 * w + lane_off, dp);
        tmem_ld_wait();
        reg_fence(s);
        reg_fence(dp);
        const float* lse2 = reinterpret_cast<const float*>(gbase + L::kRow + st * 512) + 32 * w;
        const float* Dv =
            reinterpret_cast<const float*>(gbase + L::kRow + st * 512 + 256) + 32 * w;
        const int qbase = 64 * qi + 32 * w;
        const bool need_mask = (CAUSAL && qbase + p.off < U.k0 + 127) || (qbase + 32 > p.N) ||
                               (U.k0 + 128 > p.N_kv);
        uint32_t pk[16], dsk[16];
        const uint64_t sl2x2 = f2_pack(sl2, sl2);
        // Dropout keep bits of this key for the 32 queries: the quad's four lanes (keys 4J..4J+3)
        // run two generator calls each (blocks of queries 4n..4n+3 for n = lane%4 and 4 + lane%4),
        // transpose each block's bytes so that word t holds key t's four bytes, and swap words:
        // kbits[h][g] then holds queries qbase + 16h + 4g + (0..3) of this key.
        uint32_t kbits[2][4];
        if constexpr (DROPOUT) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t wv[4] = {static_cast<uint32_t>(key) >> 2,
                              static_cast<uint32_t>((qbase >> 2) + 4 * h + (lane & 3)),
                              static_cast<uint32_t>(qh), p.drop.offset};
            philox4x32_10(wv, p.drop.seed_lo, p.drop.seed_hi);
            byte_transpose(wv, kbits[h]);
            quad_transpose(kbits[h], lane);
#pragma unroll
            for (int g = 0; g < 4; ++g) kbits[h][g] = keep_bytes(kbits[h][g], p.drop.add4);
          }
        }
        const uint64_t rk2 = f2_pack(p.drop.keep_scale, p.drop.keep_scale);
#pragma unroll
        for (int c = 0; c < 32; c += 4) {
          const float4 l4 = *reinterpret_cast<const float4*>(lse2 + c);  // -lse * log2(e)
          const float4 d4 = *reinterpret_cast<const float4*>(Dv + c);
          float a[4], pr[4], dsr[4];
          f2_unpack(f2_fma(f2_pack_u(s[c], s[c + 1]), sl2x2, f2_pack(l4.x, l4.y)), a[0], a[1]);
          f2_unpack(f2_fma(f2_pack_u(s[c + 2], s[c + 3]), sl2x2, f2_pack(l4.z, l4.w)), a[2], a[3]);
#pragma unroll
          for (int e = 0; e < 4; ++e) pr[e] = ex2_approx(a[e]);
          if constexpr (!DROPOUT) {
            f2_unpack(f2_mul(f2_pack(pr[0], pr[1]),
                             f2_sub(f2_pack_u(dp[c], dp[c + 1]), f2_pack(d4.x, d4.y))),
                      dsr[0], dsr[1]);
            f2_unpack(f2_mul(f2_pack(pr[2], pr[3]),
                             f2_sub(f2_pack_u(dp[c + 2], dp[c + 3]), f2_pack(d4.z, d4.w))),
                      dsr[2], dsr[3]);
          } else {
            // dS = P o (r Z o dP - D); the P fed to the dV MMA is Z o P (r is applied to dV at
            // the end)
            const uint32_t kb = kbits[c / 16][(c / 4) & 3];
            const uint32_t m0 = elem_mask<0>(kb), m1 = elem_mask<1>(kb);
            const uint32_t m2 = elem_mask<2>(kb), m3 = elem_mask<3>(kb);
            f2_unpack(f2_mul(f2_pack(pr[0], pr[1]),
                             f2_fma(f2_pack_u(dp[c] & m0, dp[c + 1] & m1), rk2,
                                    f2_pack(-d4.x, -d4.y))),
                      dsr[0], dsr[1]);
            f2_unpack(f2_mul(f2_pack(pr[2], pr[3]),
                             f2_fma(f2_pack_u(dp[c + 2] & m2, dp[c + 3] & m3), rk2,
                                    f2_pack(-d4.z, -d4.w))),
                      dsr[2], dsr[3]);
            pr[0] = __uint_as_float(__float_as_uint(pr[0]) & m0);
            pr[1] = __uint_as_float(__float_as_uint(pr[1]) & m1);
            pr[2] = __uint_as_float(__float_as_uint(pr[2]) & m2);
            pr[3] = __uint_as_float(__float_as_uint(pr[3]) & m3);
          }
          if (need_mask) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int q = qbase + c + e;
              if (q >= p.N || key >= p.N_kv || (CAUSAL && q + p.off < key)) {
                pr[e] = 0.f;
                dsr[e] = 0.f;
              }
            }
          }
          pk[c / 2] = pack_bf16x2(pr[0], pr[1]);
          pk[c / 2 + 1] = pack_bf16x2(pr[2], pr[3]);
          dsk[c / 2] = pack_bf16x2(dsr[0], dsr[1]);
          dsk[c / 2 + 1] = pack_bf16x2(dsr[2], dsr[3]);
        }
        tmem_st_32x32b_x16(tmem + L::tS(b) + 32 * w + lane_off, pk);
        uint8_t* dsb = gbase + L::kDS + b * 16384;
#pragma unroll
        for (int t = 0; t < 4; ++t)
          *reinterpret_cast<uint4*>(dsb + sw128_offset(r, 4 * w + t)) =
              make_uint4(dsk[4 * t], dsk[4 * t + 1], dsk[4 * t + 2], dsk[4 * t + 3]);
        tmem_st_wait();
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(bar(L::bEwDone + b));
      }
    }
    if (!ok) fail(p.status, abort_flag, 5);
  } else if (warp < 12) {
    // ------------------------------------------ dQ drain, and the unit's dK / dV -----------
    const int wq = warp & 3;                         // d columns [32 wq, 32 wq + 32)
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    float* stagef = reinterpret_cast<float*>(gbase + L::kDQ + wq * 8192);
    uint8_t* stageb = gbase + L::kDQ + wq * 8192;
    const uint32_t stage_s = sbase + L::kDQ + wq * 8192;
    const bool active = 32 * wq < p.d;
    const float scale = p.scale;
    const float dv_mul = DROPOUT ? p.drop.keep_scale : 1.0f;  // dV = r (Z o P)^T dO
    bool ok = true;
    int g = 0, uc = 0;  // tiles of earlier units; earlier units with at least one tile
    for (int si = 0; ok; ++si) {
      const int u = warp_next_unit(si);
      if (u == kGaveUp) { ok = false; break; }
      if (u < 0) break;
      const Unit U = unit_of(u);
      for (int i = 0; i < U.n_i; ++i, ++g) {
        const int b = g & 1;
        if (!warp_wait(bar(L::bDQFull + b), (g >> 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        uint32_t v[64];
        tmem_ld_32x32b_x32(tmem + L::tDP(b) + lane_off, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
        tmem_ld_32x32b_x32(tmem + L::tDP(b) + 32 + lane_off, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
        tmem_ld_wait();
        reg_fence(v);
        tc_fence_before();
        mbar_arrive(bar(L::bDQFree + b));
        if (!active) continue;
        const int qi = U.qi0 + i % U.n_qt, qh = U.bh * p.qgroup + i / U.n_qt;
        if (lane == 0) bulk_wait_group_read0();  // previous bulk copy finished reading staging
        __syncwarp();
#pragma unroll
        for (int q = 0; q < 64; ++q) stagef[q * 32 + lane] = __uint_as_float(v[q]) * scale;
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_reduce_add_3d(&tmDQacc, stage_s, 32 * wq, 64 * qi, qh);
          bulk_commit_group();
        }
      }
      if (!ok) break;
      // dV and dK * scale of the unit (zero when no query sees its keys): TMEM -> bf16 ->
      // staging (32 rows x 64 columns per 4 KB box, 128-byte swizzle) -> TMA store; at d = 128
      // dK reuses dV's staging once dV's store has read it, and TMEM is released after dK.
      const bool has = U.n_i > 0;
      if (has) {
        if (!warp_wait(bar(L::bAccDone), uc & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
      }
      const int row0 = U.k0 + 32 * wq;
      // one accumulator (TMEM columns tcol) times mul into the staging at byte offset soff
      auto stage_acc = [&](uint32_t tcol, float mul, int soff) {
#pragma unroll
        for (int c = 0; c < D; c += 32) {
          uint32_t v[32];
          if (has) {
            tmem_ld_32x32b_x32(tmem + tcol + c + lane_off, v);
            tmem_ld_wait();
            reg_fence(v);
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = 0u;
          }
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int chunk = c / 8 + q;
            *reinterpret_cast<uint4*>(stageb + soff + (chunk >> 3) * 4096 +
                                      sw128_offset(lane, chunk & 7)) =
                make_uint4(pack_bf16x2(__uint_as_float(v[8 * q]) * mul, __uint_as_float(v[8 * q + 1]) * mul),
                           pack_bf16x2(__uint_as_float(v[8 * q + 2]) * mul, __uint_as_float(v[8 * q + 3]) * mul),
                           pack_bf16x2(__uint_as_float(v[8 * q + 4]) * mul, __uint_as_float(v[8 * q + 5]) * mul),
                           pack_bf16x2(__uint_as_float(v[8 * q + 6]) * mul, __uint_as_float(v[8 * q + 7]) * mul));
          }
        }
      };
      auto store_acc = [&](const CUtensorMap* map, int soff) {
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
#pragma unroll
          for (int bx = 0; bx < L::kBoxes; ++bx)
            tma_store_3d(map, stage_s + soff + bx * 4096, 64 * bx, row0, U.bh);
          bulk_commit_group();
        }
      };
      // at d = 64 dV and dK sit side by side in the 8 KB; at d = 128 dK reuses dV's space
      constexpr int kDKOff = D == 64 ? 4096 : 0;
      if (lane == 0) bulk_wait_group_read0();
      __syncwarp();
      stage_acc(L::tDV, dv_mul, 0);
      store_acc(&tmDV, 0);
      if constexpr (D == 128) {
        if (lane == 0) bulk_wait_group_read0();
        __syncwarp();
      }
      stage_acc(L::tDK, scale, kDKOff);
      if (has) {
        tc_fence_before();
        mbar_arrive(bar(L::bAccFree));
        ++uc;
      }
      store_acc(&tmDK, kDKOff);
    }
    if (!ok) fail(p.status, abort_flag, 5);
    if (lane == 0) bulk_wait_group0();
  } else if (warp == 12) {
    // --------------------------------------------------------------------- MMA ----------
    if (lane == 0) {
      const uint32_t id_s = idesc_bf16_f32(128, 64, false, false);   // S^T, dP^T
      const uint32_t id_acc = idesc_bf16_f32(128, D, false, true);   // dV, dK
      const uint32_t id_dq = idesc_bf16_f32(128, 64, true, true);    // dQ^T
      // Operand descriptors are built once; per stage/buffer and k-step they are advanced by
      // byte offsets (see sdesc_advance).
      const uint64_t dK_k = sdesc_sw128(sbase + L::kK, 16, 1024);          // K, K-major
      const uint64_t dV_k = sdesc_sw128(sbase + L::kV, 16, 1024);          // V, K-major
      const uint64_t dKt_mn =                                              // K^T, MN-major
          sdesc_sw128(sbase + L::kK, D == 128 ? static_cast<uint32_t>(L::kKVBox) : 0u, 1024);
      const uint64_t dQ_k = sdesc_sw128(sbase + L::kQ, 16, 1024);          // Q, K-major
      const uint64_t dDO_k = sdesc_sw128(sbase + L::kDO, 16, 1024);        // dO, K-major
      const uint64_t dQ_mn = sdesc_sw128(sbase + L::kQ, L::kQBox, 1024);   // Q, MN-major
      const uint64_t dDO_mn = sdesc_sw128(sbase + L::kDO, L::kQBox, 1024); // dO, MN-major
      const uint64_t dDS = sdesc_sw128(sbase + L::kDS, 16, 1024);          // dS^T (K- or MN-major)
      auto first_half = [&](int i) {
        const int b = i & 1;
        const uint32_t so = static_cast<uint32_t>(i % QS) * 2 * L::kQTile;
        const uint64_t q0 = sdesc_advance(dQ_k, so), o0 = sdesc_advance(dDO_k, so);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t okv = (kk >> 2) * L::kKVBox + (kk & 3) * 32;
          const uint32_t oq = (kk >> 2) * L::kQBox + (kk & 3) * 32;
          umma_ss(tmem + L::tS(b), sdesc_advance(dK_k, okv), sdesc_advance(q0, oq), id_s,
                  kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t okv = (kk >> 2) * L::kKVBox + (kk & 3) * 32;
          const uint32_t oq = (kk >> 2) * L::kQBox + (kk & 3) * 32;
          umma_ss(tmem + L::tDP(b), sdesc_advance(dV_k, okv), sdesc_advance(o0, oq), id_s,
                  kk > 0 ? 1u : 0u);
        }
        umma_commit(bar(L::bSdPFull + b));
      };
      auto second_half = [&](int i, bool acc_prev) {
        const int b = i & 1, st = i % QS;
        const uint32_t so = static_cast<uint32_t>(st) * 2 * L::kQTile;
        const uint64_t qmn = sdesc_advance(dQ_mn, so), omn = sdesc_advance(dDO_mn, so);
        const uint64_t ds = sdesc_advance(dDS, b * 16384);
        const uint32_t acc = acc_prev ? 1u : 0u;  // dV, dK accumulate after the unit's first
        // dV += P^T dO: P^T (keys x 64 queries) from TMEM; query columns 0-31 were packed into
        // S columns [0,16), 32-63 into [32,48).
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_ts(tmem + L::tDV, tmem + L::tS(b) + (kk >> 1) * 32 + (kk & 1) * 8,
                  sdesc_advance(omn, kk * 2048), id_acc, kk > 0 ? 1u : acc);
        // dK += dS^T Q
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_ss(tmem + L::tDK, sdesc_advance(ds, kk * 32), sdesc_advance(qmn, kk * 2048), id_acc,
                  kk > 0 ? 1u : acc);
        // dQ^T = K^T dS^T  (M = 128 rows of d; for d = 64 the second half of the rows repeats
        // the first and is ignored by the drain)
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_ss(tmem + L::tDP(b), sdesc_advance(dKt_mn, kk * 2048), sdesc_advance(ds, kk * 2048),
                  id_dq, kk > 0 ? 1u : 0u);
        umma_commit(bar(L::bDQFull + b));
        umma_commit(bar(L::bQEmpty + st));
        umma_commit(bar(L::bDSFree + b));
      };
      const uint64_t lim = p.limit_ns;
      bool ok = true;
      int g = 0, uc = 0;  // tiles of earlier units; earlier units with at least one tile
      for (int si = 0; ok; ++si) {
        if (!(ok = mbar_wait(bar(L::bSchedFull + (si & 1)), (si >> 1) & 1, abort_flag, lim))) break;
        const int u = sched[si & 1];
        mbar_arrive(bar(L::bSchedEmpty + (si & 1)));
        if (u < 0) break;
        const int n_i = unit_of(u).n_i;
        if (n_i == 0) continue;
        if (!(ok = mbar_wait(bar(L::bKV), uc & 1, abort_flag, lim))) break;
        // the unit's first dV/dK products overwrite TMEM the previous unit's epilogue reads
        auto second = [&](int i) -> bool {
          const int gi = g + i;
          if (!mbar_wait(bar(L::bEwDone + (gi & 1)), (gi >> 1) & 1, abort_flag, lim)) return false;
          if (i == 0 && uc > 0 && !mbar_wait(bar(L::bAccFree), (uc - 1) & 1, abort_flag, lim))
            return false;
          tc_fence_after();
          second_half(gi, i > 0);
          return true;
        };
        for (int i = 0; i < n_i && ok; ++i) {
          const int gi = g + i, b = gi & 1, st = gi % QS;
          ok = mbar_wait(bar(L::bQFull + st), (gi / QS) & 1, abort_flag, lim) &&
               (gi < 2 || mbar_wait(bar(L::bDQFree + b), ((gi >> 1) & 1) ^ 1, abort_flag, lim));
          if (!ok) break;
          tc_fence_after();
          first_half(gi);
          if (i > 0) ok = second(i - 1);
        }
        if (ok) ok = second(n_i - 1);
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
    }
  } else if (warp == 13) {
    // ---------------------------------------------------- TMA, and the unit scheduler -----
    if (lane == 0) {
      bool ok = true;
      int g = 0, uc = 0;
      int issued = 0, skipped = -1, kv_loads = 0;
      int u = static_cast<int>(blockIdx.x);
      for (int si = 0;; ++si) {
        // publish unit si of this CTA (-1 when none is left) once every reader took unit si-2
        if (!mbar_wait(bar(L::bSchedEmpty + (si & 1)), ((si >> 1) & 1) ^ 1, abort_flag)) {
          ok = false;
          break;
        }
        const int pub = u < p.n_units ? u : -1;
        sched[si & 1] = pub;
        mbar_arrive(bar(L::bSchedFull + (si & 1)));
        if (pub < 0) break;
        const Unit U = unit_of(u);
        for (int i = 0; i < U.n_i; ++i) {
          const int gi = g + i, st = gi % QS;
          if (!mbar_wait(bar(L::bQEmpty + st), ((gi / QS) & 1) ^ 1, abort_flag)) {
            ok = false;
            break;
          }
          const int q0 = 64 * (U.qi0 + i % U.n_qt), qh = U.bh * p.qgroup + i / U.n_qt;
          issued = gi + 1;
          if (i == p.dbg_skip) {  // (the test hook leaves this tile out)
            skipped = gi;
          } else {
            mbar_arrive_expect_tx(bar(L::bQFull + st), 2 * L::kQTile + 512);
#pragma unroll
            for (int bx = 0; bx < L::kBoxes; ++bx) {
              tma_load_3d(sbase + L::kQ + st * 2 * L::kQTile + bx * L::kQBox, &tmQ,
                          bar(L::bQFull + st), 64 * bx, q0, qh);
              tma_load_3d(sbase + L::kDO + st * 2 * L::kQTile + bx * L::kQBox, &tmDO,
                          bar(L::bQFull + st), 64 * bx, q0, qh);
            }
            tma_load_3d(sbase + L::kRow + st * 512, &tmLse2, bar(L::bQFull + st), q0, qh, 0);
            tma_load_3d(sbase + L::kRow + st * 512 + 256, &tmD, bar(L::bQFull + st), q0, qh, 0);
          }
          if (i == 0) {
            // K and V of the unit, once every product of the previous unit has completed
            if (uc > 0 && !mbar_wait(bar(L::bAccDone), (uc - 1) & 1, abort_flag)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(bar(L::bKV), 2 * L::kKVTile);
#pragma unroll
            for (int bx = 0; bx < L::kBoxes; ++bx) {
              tma_load_3d(sbase + L::kK + bx * L::kKVBox, &tmK, bar(L::bKV), 64 * bx, U.k0, U.bh);
              tma_load_3d(sbase + L::kV + bx * L::kKVBox, &tmV, bar(L::bKV), 64 * bx, U.k0, U.bh);
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
      // gives up; the last QS loads are the latest in their stages, so on the normal path these
      // bounded waits return at once.
      volatile int never = 0;
      for (int i = max(0, issued - QS); i < issued; ++i)
        if (i != skipped) mbar_wait(bar(L::bQFull + (i % QS)), (i / QS) & 1, &never);
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

// Gate scores on the 5th-generation tensor cores ("TokenGate and T2Quant: a
// close reading", §4.1 Gate module):
//     s_j = w2 . SiLU(W1 RMSNorm(h_j) + b1) + b2   for prunable j, 0 otherwise
// with (h_j * w_n) W1^T = h_j (W1 diag(w_n))^T, so the RMSNorm weight is folded
// into W1 on the host side and the row scale 1/rms(h_j) is applied to the
// accumulator in the epilogue.  The hidden states are read from HBM once, and
// into the SM once.
//
// A persistent kernel: one CTA per SM walks the 128-token tiles t = blockIdx.x,
// blockIdx.x + gridDim.x, ...  TMA streams 128x64 tiles of H and BNx64 tiles of
// W1 (128-byte swizzle) through a STAGES-deep ring that runs on across tile
// boundaries; one thread issues tcgen05.mma (M=128, N=BN, K=16) into one of
// two fp32 TMEM accumulators (2 x BN columns), so the epilogue of tile i runs
// while the MMAs of tile i+1 stream.  Four row-norm warps sum h^2 of the
// tile's rows from the same shared-memory stages (one thread per row; the
// swizzle only permutes the 16-byte chunks inside a row's 128-byte line, which
// a sum does not see); a stage goes back to the producer once the MMAs and
// these warps have both read it.  Eight epilogue warps, two per TMEM lane
// quarter, each take half of a row's BN accumulator columns, apply 1/rms, b1,
// SiLU and w2, and the halves are added through shared memory.  Sum over
// prunable rows of s^2: per CTA over its tiles in order, then over the CTAs in
// a fixed order by the last CTA to finish (deterministic).
//
// Warp roles (448 threads): warp 0 TMA producer, warp 1 TMEM allocator + MMA
// issuer, warps 2-5 row norms, warps 6-13 epilogue (warp w reads TMEM lanes
// 32*(w%4)..+31).
#pragma once

#include "common.cuh"

namespace tg {

constexpr int kGateBM = 128;
constexpr int kGateBK = 64;
constexpr int kGateThreads = 448;
constexpr int kGateStages = 4;

struct GateParams {
  int M, N, K;        // tokens, gate hidden width h, d_model
  const __nv_bfloat16* hidden;
  const float* b1;
  const float* w2;
  float b2;
  float norm_eps;
  const uint8_t* prunable;
  float* scores;
  float* partials;    // [gridDim.x]
  uint32_t* counter;  // zero on entry
  float* sumsq;
  uint32_t* key_hist; // [2048] or null: counts of order_key(s) >> 21 over prunable tokens, zero on entry
};

constexpr int kGateHistBins = 2048;

template <int BN>
struct GateCfg {
  static constexpr int kABytes = kGateBM * kGateBK * 2;
  static constexpr int kBBytes = BN * kGateBK * 2;
  static constexpr int kBBox = BN < 128 ? BN : 128;  // rows per W1 TMA box
  static constexpr int kAccCols = BN <= 32 ? 32 : (BN <= 64 ? 64 : (BN <= 128 ? 128 : 256));
  static constexpr int kTmemCols = 2 * kAccCols;   // two accumulators
  static constexpr size_t kSmem =
      1024 + kGateStages * (kABytes + kBBytes) + 256 + 2 * BN * 4 + 2 * 2 * 128 * 4 + 64 + kGateHistBins * 4;
};

template <int BN>
__global__ void __launch_bounds__(kGateThreads, 1)
    k_gate_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
              GateParams p) {
  using Cfg = GateCfg<BN>;
  constexpr int STAGES = kGateStages;
  extern __shared__ uint8_t gate_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(gate_smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * Cfg::kABytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + STAGES * Cfg::kBBytes);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;   // [2] accumulator b holds a finished tile
  uint64_t* acc_empty = acc_full + 2;    // [2] the epilogue has read accumulator b (256 arrivals)
  uint64_t* ss_full = acc_empty + 2;     // [2] row sums of squares of the tile in buffer b (128 arrivals)
  uint64_t* ss_free = ss_full + 2;       // [2] the epilogue has read them (256 arrivals)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ss_free + 2);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  float* s_b1 = reinterpret_cast<float*>(smem + STAGES * (Cfg::kABytes + Cfg::kBBytes) + 256);
  float* s_w2 = s_b1 + BN;
  float* s_ss = s_w2 + BN;        // [2][128] row sums of h^2 per tile parity
  float* s_half = s_ss + 2 * 128; // [2][128] second-half partial dot products
  float* s_red = s_half + 2 * 128;  // 4 warp partials + broadcast slot
  uint32_t* s_hist = reinterpret_cast<uint32_t*>(s_red + 16);  // [kGateHistBins] this CTA's key histogram

  __shared__ int s_stop[2];  // [tile parity] an epilogue warp saw its wait fail
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int num_k = (p.K + kGateBK - 1) / kGateBK;
  const int tiles = (p.M + kGateBM - 1) / kGateBM;
  // this CTA's tiles: blockIdx.x, blockIdx.x + gridDim.x, ...
  const int my_tiles = blockIdx.x < tiles ? (tiles - 1 - static_cast<int>(blockIdx.x)) / gridDim.x + 1 : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1 + 4);  // the MMA commit and the four row-norm warps
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 256);
      mbar_init(&ss_full[b], 128);
      mbar_init(&ss_free[b], 256);
    }
    *abort_flag = 0;
    s_stop[0] = s_stop[1] = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();
  pdl_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (runs across tiles)
    if (lane == 0) {
      prefetch_tmap(&tmA);
      prefetch_tmap(&tmB);
      int g = 0;  // k-steps issued so far
      for (int i = 0; i < my_tiles && !*abort_flag; ++i) {
        const int tile = blockIdx.x + i * gridDim.x;
        // Every CTA needs all of W1: walking K from a tile-dependent start
        // spreads the concurrent W1 reads over different L2 lines instead of
        // having every SM hit the same k-tile at once.  (Only the fp32
        // summation order changes.)
        const int kofs = tile % num_k;
        for (int kt = 0; kt < num_k; ++kt, ++g) {
          const int s = g % STAGES;
          const uint32_t ph = (g / STAGES) & 1;
          if (!mbar_wait(&empty[s], ph ^ 1, kErrWaitGemm)) {
            *abort_flag = 1;
            break;
          }
          const int kx = ((kt + kofs) % num_k) * kGateBK;
          mbar_arrive_expect_tx(&full[s], Cfg::kABytes + Cfg::kBBytes);
          tma_load_2d(sA + s * Cfg::kABytes, &tmA, &full[s], kx, tile * kGateBM);
#pragma unroll
          for (int hb = 0; hb < BN / Cfg::kBBox; ++hb)
            tma_load_2d(sB + s * Cfg::kBBytes + hb * Cfg::kBBox * 128, &tmB, &full[s], kx, hb * Cfg::kBBox);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kGateBM, BN, false, false);
      int g = 0;
      bool ok = true;
      for (int i = 0; i < my_tiles && ok; ++i) {
        const int b = i & 1;
        // accumulator b last held tile i - 2: free once its epilogue read it
        if (i >= 2 && !(ok = mbar_wait(&acc_empty[b], ((i - 2) >> 1) & 1, kErrWaitGemm))) break;
        tc_fence_after();
        const uint32_t acc = tmem + b * Cfg::kAccCols;
        for (int kt = 0; kt < num_k; ++kt, ++g) {
          const int s = g % STAGES;
          const uint32_t ph = (g / STAGES) & 1;
          if (*abort_flag || !mbar_wait(&full[s], ph, kErrWaitGemm)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + s * Cfg::kABytes);
          const uint32_t b0 = smem_u32(sB + s * Cfg::kBBytes);
#pragma unroll
          for (int kk = 0; kk < kGateBK / 16; ++kk)
            umma_ss(acc, sdesc_sw128(a0 + kk * 32, 16, 1024), sdesc_sw128(b0 + kk * 32, 16, 1024), idesc,
                    (kt | kk) != 0 ? 1u : 0u);
          umma_commit(&empty[s]);
        }
        if (ok) umma_commit(&acc_full[b]);
      }
      if (!ok) *abort_flag = 1;
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ row norms (one thread per row)
    // Thread `row` reads its row's 128-byte line of each H stage: eight
    // 16-byte chunks, started at a row-dependent chunk so that a quarter-warp
    // touches different bank groups.
    const int row = (warp - 2) * 32 + lane;
    int g = 0;
    for (int i = 0; i < my_tiles; ++i) {
      const int b = i & 1;
      float ss = 0.0f;
      bool ok = true;
      for (int kt = 0; kt < num_k; ++kt, ++g) {
        const int s = g % STAGES;
        const uint32_t ph = (g / STAGES) & 1;
        if (*abort_flag || !warp_wait(&full[s], ph, kErrWaitGemm)) {
          ok = false;
          break;
        }
        const uint8_t* line = sA + s * Cfg::kABytes + row * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 v = *reinterpret_cast<const uint4*>(line + (((c + row) & 7) << 4));
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            ss = fmaf(bf16_lo(w[t]), bf16_lo(w[t]), ss);
            ss = fmaf(bf16_hi(w[t]), bf16_hi(w[t]), ss);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);  // release: the reads above come first
      }
      if (!ok) {
        *abort_flag = 1;
        break;
      }
      // s_ss[b] last held tile i - 2: free once its epilogue read it
      if (i >= 2 && !warp_wait(&ss_free[b], ((i - 2) >> 1) & 1, kErrWaitGemm)) {
        *abort_flag = 1;
        break;
      }
      s_ss[b * 128 + row] = ss;
      mbar_arrive(&ss_full[b]);
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 6-13)
    const int q = warp & 3;
    const int half = (warp - 6) >> 2;  // 0: columns [0, BN/2), 1: [BN/2, BN)
    const int row = q * 32 + lane;
    const int et = threadIdx.x - 6 * 32;  // 0 .. 255
    const uint32_t t_row = tmem + (static_cast<uint32_t>(q * 32) << 16);
    // columns past h (zero rows of W1 from the TMA bounds fill) contribute nothing
    for (int c = et; c < BN; c += 256) {
      s_b1[c] = (c < p.N && p.b1) ? p.b1[c] : 0.0f;
      s_w2[c] = c < p.N ? p.w2[c] : 0.0f;
    }
    if (p.key_hist)
      for (int c = et; c < kGateHistBins; c += 256) s_hist[c] = 0u;
    asm volatile("bar.sync 1, 256;" ::: "memory");
    float cta_sq = 0.0f;  // this CTA's sum of s^2, tile by tile in order (thread 0 of the group)
    bool stopped = false;
    for (int i = 0; i < my_tiles; ++i) {
      const int b = i & 1;
      const int tile = blockIdx.x + i * gridDim.x;
      const int grow = tile * kGateBM + row;
      const uint32_t ph = (i >> 1) & 1;
      const bool ok = !*abort_flag && warp_wait(&acc_full[b], ph, kErrWaitGemm) && warp_wait(&ss_full[b], ph, kErrWaitGemm);
      // all eight warps take the same decision: a warp whose wait failed sets
      // the tile's stop flag (only ever set) before the barrier, every warp
      // reads it after
      if (!ok && lane == 0) s_stop[b] = 1;
      asm volatile("bar.sync 1, 256;" ::: "memory");
      if (s_stop[b]) {
        *abort_flag = 1;
        stopped = true;
        break;
      }
      const float inv = 1.0f / sqrtf(s_ss[b * 128 + row] / static_cast<float>(p.K) + p.norm_eps);
      mbar_arrive(&ss_free[b]);
      tc_fence_after();
      float acc = 0.0f;
#pragma unroll 1
      for (int c0 = half * (BN / 2); c0 < (half + 1) * (BN / 2); c0 += 32) {
        uint32_t r[32];
        tmem_ld32(t_row + b * Cfg::kAccCols + c0, r);
        tmem_ld_wait();
#pragma unroll
        for (int t = 0; t < 32; ++t) {
          const float uval = fmaf(__uint_as_float(r[t]), inv, s_b1[c0 + t]);
          acc = fmaf(s_w2[c0 + t], __fdividef(uval, 1.0f + __expf(-uval)), acc);
        }
      }
      // accumulator b is read: the MMAs of tile i + 2 may overwrite it
      tc_fence_before();
      mbar_arrive(&acc_empty[b]);
      if (half == 1) s_half[b * 128 + row] = acc;
      asm volatile("bar.sync 1, 256;" ::: "memory");
      if (half == 0) {
        float s = 0.0f;
        bool pr = false;
        if (grow < p.M) {
          pr = p.prunable[grow] != 0;
          s = pr ? (acc + s_half[b * 128 + row]) + p.b2 : 0.0f;
          p.scores[grow] = s;
        }
        if (p.key_hist) {
          // the selector's first radix digit (key bits 31..21) over prunable
          // tokens; lanes holding the same digit add once
          const uint32_t bin = pr ? (order_key(s) >> 21) : 0xffffffffu;
          const uint32_t peers = __match_any_sync(0xffffffffu, bin);
          if (pr && lane == __ffs(peers) - 1) atomicAdd(&s_hist[bin], static_cast<uint32_t>(__popc(peers)));
        }
        // fixed-order reduction of s^2 over this tile's rows, added to the
        // CTA's running sum in tile order
        float sq = s * s;
#pragma unroll
        for (int o = 16; o; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
        if (lane == 0) s_red[q] = sq;
        asm volatile("bar.sync 2, 128;" ::: "memory");
        if (row == 0) cta_sq += (s_red[0] + s_red[1]) + (s_red[2] + s_red[3]);
        asm volatile("bar.sync 2, 128;" ::: "memory");
      }
    }
    if (p.key_hist && !stopped) {
      // this CTA's histogram into the global one (integer adds: the order does not matter)
      asm volatile("bar.sync 1, 256;" ::: "memory");
      for (int c = et; c < kGateHistBins; c += 256)
        if (s_hist[c]) atomicAdd(&p.key_hist[c], s_hist[c]);
    }
    if (half == 0 && !stopped) {
      if (row == 0) {
        p.partials[blockIdx.x] = cta_sq;
        __threadfence();
        const uint32_t prev = atomicAdd(p.counter, 1u);
        s_red[4] = (prev == gridDim.x - 1) ? 1.0f : 0.0f;
      }
      asm volatile("bar.sync 2, 128;" ::: "memory");
      if (s_red[4] != 0.0f) {
        // last CTA: sum the per-CTA partials in a fixed order
        __threadfence();
        float v = 0.0f;
        for (int i = row; i < static_cast<int>(gridDim.x); i += 128) v += __ldcg(p.partials + i);
#pragma unroll
        for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) s_red[q] = v;
        asm volatile("bar.sync 2, 128;" ::: "memory");
        if (row == 0) {
          p.sumsq[0] = (s_red[0] + s_red[1]) + (s_red[2] + s_red[3]);
          *p.counter = 0u;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    __syncwarp();  // the .sync.aligned dealloc needs the whole warp converged
    tmem_dealloc(tmem, Cfg::kTmemCols);
  }
}

}  // namespace tg

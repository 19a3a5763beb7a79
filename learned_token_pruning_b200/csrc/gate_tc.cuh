// Gate scores on the 5th-generation tensor cores ("TokenGate and T2Quant: a
// close reading", §4.1 Gate module):
//     s_j = w2 . SiLU(W1 RMSNorm(h_j) + b1) + b2   for prunable j, 0 otherwise
// with (h_j * w_n) W1^T = h_j (W1 diag(w_n))^T, so the RMSNorm weight is folded
// into W1 on the host side and the row scale 1/rms(h_j) is applied to the
// accumulator in the epilogue.  The hidden states are read from HBM once, and
// into the SM once.
//
// One CTA scores 128 tokens.  TMA streams 128x64 tiles of H and BNx64 tiles of
// W1 (128-byte swizzle) through a STAGES-deep ring; one thread issues
// tcgen05.mma (M=128, N=BN, K=16) into an fp32 TMEM accumulator.  While the
// MMAs run, the eight epilogue warps sum h^2 of the CTA's rows from the same
// shared-memory tiles (two threads per row, 64 bytes each per tile: the
// swizzle only permutes the 16-byte chunks inside a row's 128-byte line, which
// a sum does not see); a stage goes back to the producer once the MMAs and
// these warps have both read it.  Then the eight epilogue warps,
// two per TMEM lane quarter, each take half of a row's BN accumulator
// columns, apply 1/rms, b1, SiLU and w2, and the halves are added through
// shared memory.  Sum over prunable rows of s^2 is reduced in a fixed order
// by the last CTA to finish (deterministic).
//
// Warp roles (320 threads): warp 0 TMA producer, warp 1 TMEM allocator + MMA
// issuer, warps 2-9 row norms, then epilogue (warp w reads TMEM lanes
// 32*(w%4)..+31).
#pragma once

#include "common.cuh"

namespace tg {

constexpr int kGateBM = 128;
constexpr int kGateBK = 64;
constexpr int kGateThreads = 320;
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
};

template <int BN>
struct GateCfg {
  static constexpr int kABytes = kGateBM * kGateBK * 2;
  static constexpr int kBBytes = BN * kGateBK * 2;
  static constexpr int kBBox = BN < 128 ? BN : 128;  // rows per W1 TMA box
  static constexpr int kTmemCols = BN <= 32 ? 32 : (BN <= 64 ? 64 : (BN <= 128 ? 128 : 256));
  static constexpr size_t kSmem = 1024 + kGateStages * (kABytes + kBBytes) + 256 + 2 * BN * 4 + 2 * 128 * 4 + 64;
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
  uint64_t* accbar = empty + STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accbar + 1);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  float* s_b1 = reinterpret_cast<float*>(smem + STAGES * (Cfg::kABytes + Cfg::kBBytes) + 256);
  float* s_w2 = s_b1 + BN;
  float* s_ss = s_w2 + BN;    // [128] row sums of h^2
  float* s_half = s_ss + 128; // [128] second-half partial dot products
  float* s_red = s_half + 128;  // 4 warp partials + broadcast slot

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * kGateBM;
  const int num_k = (p.K + kGateBK - 1) / kGateBK;
  // Every CTA needs all of W1: walking K from a CTA-dependent start spreads
  // the concurrent W1 reads over different L2 lines instead of having every
  // SM hit the same k-tile at once.  (Only the fp32 summation order changes.)
  const int kofs = static_cast<int>(blockIdx.x % num_k);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1 + 8);  // the MMA commit and the eight row-norm warps
    }
    mbar_init(accbar, 1);
    *abort_flag = 0;
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
  if (threadIdx.x >= 64) {
    // columns past h (zero rows of W1 from the TMA bounds fill) contribute
    // nothing; read by the epilogue after its first named barrier
    for (int i = threadIdx.x - 64; i < BN; i += kGateThreads - 64) {
      s_b1[i] = (i < p.N && p.b1) ? p.b1[i] : 0.0f;
      s_w2[i] = i < p.N ? p.w2[i] : 0.0f;
    }
  }

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tmA);
      prefetch_tmap(&tmB);
      for (int kt = 0; kt < num_k; ++kt) {
        const int s = kt % STAGES;
        const uint32_t ph = (kt / STAGES) & 1;
        if (*abort_flag || !mbar_wait(&empty[s], ph ^ 1, kErrWaitGemm)) {
          *abort_flag = 1;
          break;
        }
        const int kx = ((kt + kofs) % num_k) * kGateBK;
        mbar_arrive_expect_tx(&full[s], Cfg::kABytes + Cfg::kBBytes);
        tma_load_2d(sA + s * Cfg::kABytes, &tmA, &full[s], kx, m0);
#pragma unroll
        for (int hb = 0; hb < BN / Cfg::kBBox; ++hb)
          tma_load_2d(sB + s * Cfg::kBBytes + hb * Cfg::kBBox * 128, &tmB, &full[s], kx, hb * Cfg::kBBox);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kGateBM, BN, false, false);
      for (int kt = 0; kt < num_k; ++kt) {
        const int s = kt % STAGES;
        const uint32_t ph = (kt / STAGES) & 1;
        if (*abort_flag || !mbar_wait(&full[s], ph, kErrWaitGemm)) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t a0 = smem_u32(sA + s * Cfg::kABytes);
        const uint32_t b0 = smem_u32(sB + s * Cfg::kBBytes);
#pragma unroll
        for (int kk = 0; kk < kGateBK / 16; ++kk)
          umma_ss(tmem, sdesc_sw128(a0 + kk * 32, 16, 1024), sdesc_sw128(b0 + kk * 32, 16, 1024), idesc,
                  (kt | kk) != 0 ? 1u : 0u);
        umma_commit(&empty[s]);
      }
      umma_commit(accbar);
    }
  } else {
    // ---------------- warps 2-9: row norms (6-9), then the epilogue (all eight)
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;  // 0: columns [0, BN/2), 1: [BN/2, BN)
    const int row = q * 32 + lane;
    const int grow = m0 + row;
    const uint32_t t_row = tmem + (static_cast<uint32_t>(q * 32) << 16);
    {
      // Row norms from the ring: thread e = threadIdx.x - 64 owns half e & 1
      // of row e >> 1 (four 16-byte chunks per tile, rotated by the row so
      // that a quarter-warp touches four different bank groups).
      const int e = threadIdx.x - 64;
      const int nrow = e >> 1, nhalf = e & 1;
      float ss = 0.0f;
      for (int kt = 0; kt < num_k; ++kt) {
        const int s = kt % STAGES;
        const uint32_t ph = (kt / STAGES) & 1;
        if (*abort_flag || !warp_wait(&full[s], ph, kErrWaitGemm)) {
          *abort_flag = 1;
          break;
        }
        const uint8_t* line = sA + s * Cfg::kABytes + nrow * 128 + nhalf * 64;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint4 v = *reinterpret_cast<const uint4*>(line + (((i + nrow) & 3) << 4));
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
      ss += __shfl_xor_sync(0xffffffffu, ss, 1);
      if (nhalf == 0) s_ss[nrow] = ss;
    }
    bool ok = !*abort_flag && warp_wait(accbar, 0, kErrWaitGemm);
    if (!ok) *abort_flag = 1;
    // all eight warps meet here (every wait above is bounded), so the abort
    // decision below is the same for all of them; the row norms are visible
    asm volatile("bar.sync 1, 256;" ::: "memory");
    if (!*abort_flag) {
      tc_fence_after();
      const float inv = 1.0f / sqrtf(s_ss[row] / static_cast<float>(p.K) + p.norm_eps);
      float acc = 0.0f;
#pragma unroll 1
      for (int c0 = half * (BN / 2); c0 < (half + 1) * (BN / 2); c0 += 32) {
        uint32_t r[32];
        tmem_ld32(t_row + c0, r);
        tmem_ld_wait();
#pragma unroll
        for (int t = 0; t < 32; ++t) {
          const float uval = fmaf(__uint_as_float(r[t]), inv, s_b1[c0 + t]);
          acc = fmaf(s_w2[c0 + t], __fdividef(uval, 1.0f + __expf(-uval)), acc);
        }
      }
      if (half == 1) s_half[row] = acc;
      asm volatile("bar.sync 1, 256;" ::: "memory");
      if (half == 0) {
        float s = 0.0f;
        if (grow < p.M) {
          s = p.prunable[grow] ? (acc + s_half[row]) + p.b2 : 0.0f;
          p.scores[grow] = s;
        }
        // fixed-order reduction of s^2 over this CTA's rows
        float sq = s * s;
#pragma unroll
        for (int o = 16; o; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
        if (lane == 0) s_red[q] = sq;
        asm volatile("bar.sync 2, 128;" ::: "memory");
        if (row == 0) {
          p.partials[blockIdx.x] = (s_red[0] + s_red[1]) + (s_red[2] + s_red[3]);
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

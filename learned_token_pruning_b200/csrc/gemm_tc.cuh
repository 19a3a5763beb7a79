// bf16 GEMM on the 5th-generation tensor cores: C[M][N] = A[M][K] * B[N][K]^T.
//
// One CTA computes a 128 x BN tile.  TMA streams 128x64 A tiles and BNx64 B
// tiles (128-byte swizzle) through a STAGES-deep shared-memory ring; a single
// thread issues tcgen05.mma (M=128, N=BN, K=16) into an fp32 accumulator held
// in tensor memory; four epilogue warps read it back with tcgen05.ld and apply
// one of the fused epilogues:
//   kEpiStore     C = acc                                 (bf16)
//   kEpiResidual  C = C + acc                             (bf16, in place)
//   kEpiSwiGLU    C[:, f] = SiLU(acc[:, f]) * acc[:, 128 + f], where the two
//                 halves of the B tile are the gate rows and the up rows of
//                 the same 128 features
//   kEpiGateScore s_row = w2 . SiLU(acc_row / rms(A_row) + b1) + b2 for
//                 prunable rows, else 0 -- the TokenGate gate MLP ("TokenGate and
//                 T2Quant: a close reading", §4.1 Gate module) with the row
//                 RMSNorm folded in: the epilogue warps accumulate sum(A_row^2)
//                 from the shared-memory A tiles while the MMAs run, so the
//                 hidden states are read from HBM exactly once.  A fixed-order
//                 last-CTA reduction produces sum over prunable rows of s^2.
//
// Warp roles (192 threads): warp 0 = TMA producer, warp 1 = TMEM allocator and
// MMA issuer, warps 2-5 = epilogue (warp w reads TMEM lanes 32*(w%4)..+31).
#pragma once

#include "common.cuh"

namespace tg {

constexpr int kGemmBM = 128;
constexpr int kGemmBK = 64;
constexpr int kGemmThreads = 192;

enum GemmEpilogue { kEpiStore = 0, kEpiResidual = 1, kEpiSwiGLU = 2, kEpiGateScore = 3 };

struct GemmParams {
  int M, N, K;
  __nv_bfloat16* out;  // store / residual / SwiGLU output
  int64_t ldo;
  int up_row0;         // SwiGLU: first B row of the up block (= d_ff)
  // gate score
  const float* b1;
  const float* w2;
  float b2;
  float norm_eps;
  const float* norm_w_unused;
  const uint8_t* prunable;
  float* scores;
  float* partials;     // [gridDim.y]
  uint32_t* counter;   // zero on entry
  float* sumsq;
};

template <int BN>
struct GemmCfg {
  static constexpr int kABytes = kGemmBM * kGemmBK * 2;
  static constexpr int kBBytes = BN * kGemmBK * 2;
  static constexpr int kBBox = BN < 128 ? BN : 128;  // rows per B TMA box
  static constexpr int kTmemCols = BN <= 32 ? 32 : (BN <= 64 ? 64 : (BN <= 128 ? 128 : 256));
};

template <int BN, int STAGES>
constexpr size_t gemm_smem_bytes() {
  return 1024 /*align*/ + STAGES * (GemmCfg<BN>::kABytes + GemmCfg<BN>::kBBytes) + 256 /*barriers*/ +
         2 * BN * 4 /*b1,w2*/ + 64;
}

template <int BN, int STAGES, int EPI>
__global__ void __launch_bounds__(kGemmThreads, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, GemmParams p) {
  using Cfg = GemmCfg<BN>;
  extern __shared__ uint8_t gemm_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(gemm_smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * Cfg::kABytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + STAGES * Cfg::kBBytes);
  uint64_t* empty = full + STAGES;
  uint64_t* accbar = empty + STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accbar + 1);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  float* s_b1 = reinterpret_cast<float*>(smem + STAGES * (Cfg::kABytes + Cfg::kBBytes) + 256);
  float* s_w2 = s_b1 + BN;
  float* s_red = s_w2 + BN;  // 4 warp partials + broadcast slot

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * kGemmBM;
  const int nb = blockIdx.x;
  const int num_k = (p.K + kGemmBK - 1) / kGemmBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], EPI == kEpiGateScore ? 1 + 4 : 1);
    }
    mbar_init(accbar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::kTmemCols);
    tmem_relinquish();
  }
  if (EPI == kEpiGateScore && threadIdx.x >= 64) {
    // columns past h (zero rows of W1 from the TMA bounds fill) contribute nothing
    for (int i = threadIdx.x - 64; i < BN; i += 128) {
      s_b1[i] = (i < p.N && p.b1) ? p.b1[i] : 0.0f;
      s_w2[i] = i < p.N ? p.w2[i] : 0.0f;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

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
        mbar_arrive_expect_tx(&full[s], Cfg::kABytes + Cfg::kBBytes);
        tma_load_2d(sA + s * Cfg::kABytes, &tmA, &full[s], kt * kGemmBK, m0);
#pragma unroll
        for (int hb = 0; hb < BN / Cfg::kBBox; ++hb) {
          const int brow = (EPI == kEpiSwiGLU) ? (hb * p.up_row0 + nb * 128) : (nb * BN + hb * Cfg::kBBox);
          tma_load_2d(sB + s * Cfg::kBBytes + hb * Cfg::kBBox * 128, &tmB, &full[s], kt * kGemmBK, brow);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kGemmBM, BN, false, false);
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
        for (int kk = 0; kk < kGemmBK / 16; ++kk) {
          umma_ss(tmem, sdesc_sw128(a0 + kk * 32, 16, 1024), sdesc_sw128(b0 + kk * 32, 16, 1024), idesc,
                  (kt | kk) != 0 ? 1u : 0u);
        }
        umma_commit(&empty[s]);
      }
      umma_commit(accbar);
    }
  } else {
    // ---------------- epilogue warps
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const int grow = m0 + row;
    const uint32_t t_row = tmem + (static_cast<uint32_t>(q * 32) << 16);
    float ss = 0.0f;
    bool ok = true;
    if (EPI == kEpiGateScore) {
      for (int kt = 0; kt < num_k; ++kt) {
        const int s = kt % STAGES;
        const uint32_t ph = (kt / STAGES) & 1;
        if (*abort_flag || !warp_wait(&full[s], ph, kErrWaitGemm)) {
          ok = false;
          *abort_flag = 1;
          break;
        }
        // the 128-byte swizzle permutes 16-byte chunks inside the row only
        const uint4* src = reinterpret_cast<const uint4*>(sA + s * Cfg::kABytes + row * 128);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 v = src[c];
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const float lo = bf16_lo(w[t]), hi = bf16_hi(w[t]);
            ss = fmaf(lo, lo, ss);
            ss = fmaf(hi, hi, ss);
          }
        }
        // order these generic-proxy reads before the TMA (async proxy) refill of the stage
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
      }
    }
    if (ok && !*abort_flag) ok = warp_wait(accbar, 0, kErrWaitGemm);
    if (!ok) *abort_flag = 1;
    // all four epilogue warps meet here (every wait above is bounded), so the
    // abort decision below is the same for all of them
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (!*abort_flag) {
      tc_fence_after();
      if (EPI == kEpiStore || EPI == kEpiResidual) {
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 32) {
          uint32_t r[32];
          tmem_ld32(t_row + c0, r);
          tmem_ld_wait();
          const int gcol = nb * BN + c0;
          if (grow < p.M && gcol < p.N) {
            uint4* dst = reinterpret_cast<uint4*>(p.out + static_cast<int64_t>(grow) * p.ldo + gcol);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              float add[8] = {0, 0, 0, 0, 0, 0, 0, 0};
              if (EPI == kEpiResidual) {
                const uint4 old = dst[v];
                const uint32_t ow[4] = {old.x, old.y, old.z, old.w};
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                  add[2 * t] = bf16_lo(ow[t]);
                  add[2 * t + 1] = bf16_hi(ow[t]);
                }
              }
              uint4 o;
              o.x = pack_bf16x2(__uint_as_float(r[8 * v + 0]) + add[0], __uint_as_float(r[8 * v + 1]) + add[1]);
              o.y = pack_bf16x2(__uint_as_float(r[8 * v + 2]) + add[2], __uint_as_float(r[8 * v + 3]) + add[3]);
              o.z = pack_bf16x2(__uint_as_float(r[8 * v + 4]) + add[4], __uint_as_float(r[8 * v + 5]) + add[5]);
              o.w = pack_bf16x2(__uint_as_float(r[8 * v + 6]) + add[6], __uint_as_float(r[8 * v + 7]) + add[7]);
              dst[v] = o;
            }
          }
        }
      } else if (EPI == kEpiSwiGLU) {
#pragma unroll 1
        for (int c0 = 0; c0 < 128; c0 += 32) {
          uint32_t g[32], u[32];
          tmem_ld32(t_row + c0, g);
          tmem_ld32(t_row + 128 + c0, u);
          tmem_ld_wait();
          const int gcol = nb * 128 + c0;
          if (grow < p.M && gcol < p.N) {
            uint4* dst = reinterpret_cast<uint4*>(p.out + static_cast<int64_t>(grow) * p.ldo + gcol);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              float a[8];
#pragma unroll
              for (int t = 0; t < 8; ++t) {
                const float gv = __uint_as_float(g[8 * v + t]);
                a[t] = gv / (1.0f + __expf(-gv)) * __uint_as_float(u[8 * v + t]);
              }
              uint4 o;
              o.x = pack_bf16x2(a[0], a[1]);
              o.y = pack_bf16x2(a[2], a[3]);
              o.z = pack_bf16x2(a[4], a[5]);
              o.w = pack_bf16x2(a[6], a[7]);
              dst[v] = o;
            }
          }
        }
      } else if (EPI == kEpiGateScore) {
        const float inv = 1.0f / sqrtf(ss / static_cast<float>(p.K) + p.norm_eps);
        float acc = 0.0f;
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 32) {
          uint32_t r[32];
          tmem_ld32(t_row + c0, r);
          tmem_ld_wait();
#pragma unroll
          for (int t = 0; t < 32; ++t) {
            const float uval = fmaf(__uint_as_float(r[t]), inv, s_b1[c0 + t]);
            acc = fmaf(s_w2[c0 + t], uval / (1.0f + expf(-uval)), acc);
          }
        }
        float s = 0.0f;
        if (grow < p.M) {
          s = p.prunable[grow] ? acc + p.b2 : 0.0f;
          p.scores[grow] = s;
        }
        // fixed-order reduction of s^2 over this CTA's rows
        float sq = s * s;
#pragma unroll
        for (int o = 16; o; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
        if (lane == 0) s_red[q] = sq;
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (row == 0) {
          const float part = (s_red[0] + s_red[1]) + (s_red[2] + s_red[3]);
          p.partials[blockIdx.y] = part;
          __threadfence();
          const uint32_t prev = atomicAdd(p.counter, 1u);
          s_red[4] = (prev == gridDim.y - 1) ? 1.0f : 0.0f;
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (s_red[4] != 0.0f) {
          // last CTA: sum the per-CTA partials in a fixed order
          __threadfence();
          float v = 0.0f;
          for (int i = row; i < static_cast<int>(gridDim.y); i += 128) v += __ldcg(p.partials + i);
#pragma unroll
          for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
          if (lane == 0) s_red[q] = v;
          asm volatile("bar.sync 1, 128;" ::: "memory");
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

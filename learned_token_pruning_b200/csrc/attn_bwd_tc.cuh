// Backward of token-gated causal GQA attention on the 5th-generation tensor
// cores ("TokenGate and T2Quant: a close reading", §4.1 engineering notes: the
// biased attention kernel also returns the bias gradient to the scorer).  The
// gradients are those of the CUDA-core kernels beside it:
//     dl_rc = P_rc (dP_rc - D_r),   dP_rc = dO_r . v_c,   D_r = dO_r . o_r
//     dS_rc = dl_rc a_r sm_scale,   a_r = temp_h ratio_r
//     dq_r = sum_c dS_rc k_c;  dk_c = sum_{h, r} dS_rc q_r;  dv_c = sum_{h, r} P_rc dO_r
//     dbias_c = sum_h gain_h sum_r dl_rc;  dgain_h = sum dl_rc bias_c;  dtemp_h = sum dl_rc ratio_r z_rc
// with P recomputed as exp2(a_r sm_scale log2(e) S_rc + gain_h log2(e) bias_c - lse_r log2(e)).
// Products that feed a tensor-core MMA (P and dS) are rounded to bf16; every
// sum is fp32; nothing is summed by atomics, so reruns are bit-identical.
//
// k_attn_bwd_dq_tc: one CTA per (query head h, block of 128 rows), walking the
//   key tiles of 64 up to the diagonal.  S = Q K^T and dP = dO V^T are SS-MMAs
//   into double-buffered tensor memory; two warpgroups (one thread per row,
//   each taking 32 of a tile's 64 keys) turn them into dS, written as bf16
//   pairs over the first 16 columns of their half of the S buffer, and the
//   MMA thread accumulates dQ += dS K as a TS-MMA (K MN-major from shared
//   memory).  The row's dgain / dtemp contributions are summed on the way.
// k_attn_bwd_kv_tc: one CTA per (KV head g, block of 128 keys), walking the
//   query tiles of 64 rows from the diagonal on, for every query head of g.
//   S^T = K Q^T and dP^T = V dO^T (one thread per key), P^T and dS^T as bf16
//   pairs over their own columns, then dV += P^T dO and dK += dS^T Q as
//   TS-MMAs; both accumulators stay in tensor memory over the whole walk.  The
//   per-row constants of a tile (from k_attn_bwd_prep) come by TMA into the
//   same stage as the Q / dO tiles.
// k_attn_bwd_prep: D_r and the per-row constants (a_r sm_scale log2 e,
//   -lse_r log2 e, D_r, a_r sm_scale) of every head and row, rows past m
//   masked (P = 0 there), so neither kernel above reads lse or ratio per tile.
//
// Warps: 0-7 elementwise (two warpgroups), 8 TMA producer, 9 TMEM allocator
// and single-thread MMA issuer.  Every wait is bounded (kErrWaitAttention).
#pragma once

#include "attn_bwd.cuh"
#include "attn_tc.cuh"
#include "common.cuh"

namespace tg {

constexpr int kBwdTcThreads = 320;

template <int D>
struct BwdDqCfg {
  static constexpr int BM = 128, BN = 64, kStages = 4;
  static constexpr int kQBytes = BM * D * 2;   // a Q or dO block (128 rows)
  static constexpr int kQBlk = BM * 128;       // one 64-column box of it
  static constexpr int kKVBytes = BN * D * 2;  // a K or V tile (64 keys)
  static constexpr int kKVBlk = BN * 128;
  static constexpr size_t kOffDO = kQBytes;
  static constexpr size_t kOffK = 2 * size_t(kQBytes);
  static constexpr size_t kOffV = kOffK + kStages * size_t(kKVBytes);
  static constexpr size_t kOffBias = kOffV + kStages * size_t(kKVBytes);
  static constexpr size_t kOffRed = kOffBias + kStages * BN * 4;  // [8 warps][2]
  static constexpr size_t kOffBars = kOffRed + 64;
  static constexpr size_t kData = kOffBars + 256;
  // one CTA per SM, so that its 512-column TMEM allocation never waits
  static constexpr size_t kSmem = 1024 + (kData < 120 * 1024 ? 120 * 1024 : kData);
  static constexpr uint32_t kColDP = 128, kColDQ = 256;  // S[b] at 64 b, dP[b] at 128 + 64 b
};

template <int D>
struct BwdKvCfg {
  static constexpr int BK = 128, BR = 64, kStages = 4;
  static constexpr int kKBytes = BK * D * 2;  // the K or V block (128 keys)
  static constexpr int kKBlk = BK * 128;
  static constexpr int kRBytes = BR * D * 2;  // a Q or dO tile (64 rows)
  static constexpr int kRBlk = BR * 128;
  static constexpr size_t kOffV = kKBytes;
  static constexpr size_t kOffQ = 2 * size_t(kKBytes);
  static constexpr size_t kOffDO = kOffQ + kStages * size_t(kRBytes);
  static constexpr size_t kOffPar = kOffDO + kStages * size_t(kRBytes);  // [stage][64 rows] float4
  static constexpr size_t kOffRed = kOffPar + kStages * BR * 16;         // [128] floats
  static constexpr size_t kOffBars = kOffRed + BK * 4;
  static constexpr size_t kData = kOffBars + 256;
  static constexpr size_t kSmem = 1024 + (kData < 120 * 1024 ? 120 * 1024 : kData);
  static constexpr uint32_t kColDP = 128, kColDV = 256, kColDK = 256 + D;
};

// TMEM column of the packed-bf16 K slice kk (16 elements) of a 64-wide tile
// whose two 32-wide halves were packed into the first 16 columns of each half
__device__ __forceinline__ uint32_t bwd_packed_col(int kk) {
  return static_cast<uint32_t>(kk < 2 ? kk * 8 : 32 + (kk - 2) * 8);
}

// ---------------------------------------------------------------------------
// Per-row constants: one warp per (row, head), rows m .. m_pad - 1 masked
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) k_attn_bwd_prep(AttnBwdParams p) {
  const int w = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (w >= p.m_pad * p.hq) return;  // warp-uniform
  const int r = w / p.hq, h = w % p.hq;
  float4* dst = p.rowpar + int64_t(h) * p.m_pad + r;
  if (r >= p.m) {
    if (lane == 0) *dst = make_float4(0.0f, -INFINITY, 0.0f, 0.0f);
    return;
  }
  const __nv_bfloat16* go = static_cast<const __nv_bfloat16*>(p.dout) + int64_t(r) * p.lddo + h * D;
  const __nv_bfloat16* oo = static_cast<const __nv_bfloat16*>(p.o) + int64_t(r) * p.ldo + h * D;
  float s = 0.0f;
  if constexpr (D == 128) {
    const uint2 a = reinterpret_cast<const uint2*>(go)[lane], b = reinterpret_cast<const uint2*>(oo)[lane];
    s = bf16_lo(a.x) * bf16_lo(b.x) + bf16_hi(a.x) * bf16_hi(b.x) + bf16_lo(a.y) * bf16_lo(b.y) +
        bf16_hi(a.y) * bf16_hi(b.y);
  } else {
    const uint32_t a = reinterpret_cast<const uint32_t*>(go)[lane], b = reinterpret_cast<const uint32_t*>(oo)[lane];
    s = bf16_lo(a) * bf16_lo(b) + bf16_hi(a) * bf16_hi(b);
  }
#pragma unroll
  for (int off = 16; off; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if (lane == 0) {
    const float as = p.temp[h] * (p.ratio ? p.ratio[r] : 1.0f) * p.sm_scale;
    *dst = make_float4(as * kLog2e, -p.lse[int64_t(h) * p.m + r] * kLog2e, s, as);
  }
}

// ---------------------------------------------------------------------------
// dQ (and the dgain / dtemp partials)
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(kBwdTcThreads, 1)
    k_attn_bwd_dq_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                     const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const __grid_constant__ CUtensorMap tmBias, AttnBwdParams p) {
  using Cfg = BwdDqCfg<D>;
  constexpr int BN = Cfg::BN;
  constexpr int kDBoxes = D / 64;
  extern __shared__ uint8_t bwd_tc_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(bwd_tc_smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sDO = smem + Cfg::kOffDO;
  uint8_t* sK = smem + Cfg::kOffK;
  uint8_t* sV = smem + Cfg::kOffV;
  float* sBias = reinterpret_cast<float*>(smem + Cfg::kOffBias);
  float* red = reinterpret_cast<float*>(smem + Cfg::kOffRed);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kOffBars);
  uint64_t* q_full = bars + 0;
  constexpr int kS = Cfg::kStages;
  uint64_t* kv_full = bars + 1;        // [kS] K, V and bias tile j (stage j % kS)
  uint64_t* dq_done = kv_full + kS;    // [kS] dQ += dS K of tile j complete: stage j % kS free
  uint64_t* s_full = dq_done + kS;     // [2] S and dP of tile j in buffer j % 2
  uint64_t* ds_full = s_full + 2;      // [2] dS of tile j written (256 arrivals)
  uint64_t* o_final = ds_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(o_final + 1);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nqb = (p.m + 127) / 128;
  // longest first: the last row blocks see the most keys
  const int qb = nqb - 1 - static_cast<int>(blockIdx.x) / p.hq;
  const int h = static_cast<int>(blockIdx.x) % p.hq;
  const int g = h / p.group;
  const int nt = min(2 * qb + 2, (p.m + BN - 1) / BN);
  const bool has_bias = p.bias != nullptr;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kS; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&dq_done[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&ds_full[b], 256);
    }
    mbar_init(o_final, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (!has_bias)
    for (int i = threadIdx.x; i < kS * BN; i += kBwdTcThreads) sBias[i] = 0.0f;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmDO);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      if (has_bias) prefetch_tmap(&tmBias);
      mbar_arrive_expect_tx(q_full, 2 * Cfg::kQBytes);
      for (int b = 0; b < kDBoxes; ++b) {
        tma_load_2d(sQ + b * Cfg::kQBlk, &tmQ, q_full, h * D + 64 * b, qb * 128);
        tma_load_2d(sDO + b * Cfg::kQBlk, &tmDO, q_full, h * D + 64 * b, qb * 128);
      }
      for (int j = 0; j < nt; ++j) {
        const int s = j % kS;
        if (j >= kS && !mbar_wait(&dq_done[s], ((j - kS) / kS) & 1, kErrWaitAttention)) {
          *abort_flag = 1;
          break;
        }
        mbar_arrive_expect_tx(&kv_full[s], 2 * Cfg::kKVBytes + (has_bias ? BN * 4 : 0));
        for (int b = 0; b < kDBoxes; ++b) {
          tma_load_2d(sK + s * Cfg::kKVBytes + b * Cfg::kKVBlk, &tmK, &kv_full[s], g * D + 64 * b, j * BN);
          tma_load_2d(sV + s * Cfg::kKVBytes + b * Cfg::kKVBlk, &tmV, &kv_full[s], g * D + 64 * b, j * BN);
        }
        if (has_bias) tma_load_1d(sBias + s * BN, &tmBias, &kv_full[s], j * BN);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, BN, false, false);
      constexpr uint32_t idesc_dq = idesc_bf16_f32(128, D, false, true);
      const uint64_t dq0 = sdesc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t ddo0 = sdesc_sw128(smem_u32(sDO), 16, 1024);
      const uint64_t dk0 = sdesc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t dv0 = sdesc_sw128(smem_u32(sV), 16, 1024);
      const uint64_t dkmn0 = sdesc_sw128(smem_u32(sK), Cfg::kKVBlk, 1024);
      auto issue_s = [&](int j) {
        const int b = j & 1, s = j % kS;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ao = ((kk >> 2) * Cfg::kQBlk + (kk & 3) * 32) >> 4;
          const uint32_t bo = (s * Cfg::kKVBytes + (kk >> 2) * Cfg::kKVBlk + (kk & 3) * 32) >> 4;
          umma_ss(tmem + 64 * b, dq0 + ao, dk0 + bo, idesc_s, kk != 0 ? 1u : 0u);
          umma_ss(tmem + Cfg::kColDP + 64 * b, ddo0 + ao, dv0 + bo, idesc_s, kk != 0 ? 1u : 0u);
        }
        umma_commit(&s_full[b]);
      };
      auto issue_dq = [&](int j) {
        const int b = j & 1, s = j % kS;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          umma_ts(tmem + Cfg::kColDQ, tmem + 64 * b + bwd_packed_col(kk),
                  dkmn0 + ((s * Cfg::kKVBytes + kk * 16 * 128) >> 4), idesc_dq, (j | kk) != 0 ? 1u : 0u);
        umma_commit(&dq_done[s]);
      };
      bool ok = mbar_wait2(q_full, 0, &kv_full[0], 0, kErrWaitAttention);
      if (ok) {
        tc_fence_after();
        issue_s(0);
      }
      if (ok && nt > 1 && (ok = mbar_wait(&kv_full[1], 0, kErrWaitAttention))) {
        tc_fence_after();
        issue_s(1);
      }
      for (int j = 0; ok && j < nt; ++j) {
        const bool next = j + 2 < nt;
        ok = mbar_wait(&ds_full[j & 1], (j >> 1) & 1, kErrWaitAttention) &&
             (!next || mbar_wait(&kv_full[(j + 2) % kS], ((j + 2) / kS) & 1, kErrWaitAttention));
        if (!ok) break;
        tc_fence_after();
        issue_dq(j);
        if (next) issue_s(j + 2);  // into the buffers dQ of tile j has just read (in issue order)
      }
      if (ok) umma_commit(o_final);
      else *abort_flag = 1;
    }
  } else {
    // ------------------------------------------------------------ elementwise warpgroups
    const int wg = warp >> 2, q4 = warp & 3;
    const int row = q4 * 32 + lane, grow = qb * 128 + row;
    const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
    const bool row_ok = grow < p.m;
    const float ratio_r = row_ok ? (p.ratio ? p.ratio[grow] : 1.0f) : 0.0f;
    const float4 pr = p.rowpar[int64_t(h) * p.m_pad + grow];  // (a2, nl, D_r, as), masked past m
    const float a2 = pr.x, nl = pr.y, dr = pr.z, as = pr.w;
    const float gg = p.gain[h] * kLog2e;
    float dgain_acc = 0.0f, dtz_acc = 0.0f;
    bool ok = true;
    for (int j = 0; j < nt; ++j) {
      const int b = j & 1;
      bool rdy = !*abort_flag &&
                 mbar_wait2(&s_full[b], (j >> 1) & 1, &kv_full[j % kS], (j / kS) & 1, kErrWaitAttention);
      if (!__all_sync(0xffffffffu, rdy)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sr[32], dp[32];
      tmem_ld32(tmem + lane_base + 64 * b + 32 * wg, sr);
      tmem_ld32(tmem + lane_base + Cfg::kColDP + 64 * b + 32 * wg, dp);
      tmem_ld_wait();
      const float* bias = sBias + (j % kS) * BN + 32 * wg;
      const int key0 = j * BN + 32 * wg;
      const bool diag = key0 + 31 > qb * 128;  // warp-uniform
      uint32_t pk[16];
#pragma unroll
      for (int e = 0; e < 32; e += 2) {
        const float s0 = __uint_as_float(sr[e]), s1 = __uint_as_float(sr[e + 1]);
        float x0 = fmaf(a2, s0, fmaf(gg, bias[e], nl));
        float x1 = fmaf(a2, s1, fmaf(gg, bias[e + 1], nl));
        if (diag) {
          if (key0 + e > grow) x0 = -INFINITY;
          if (key0 + e + 1 > grow) x1 = -INFINITY;
        }
        const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
        const float dl0 = p0 * (__uint_as_float(dp[e]) - dr);
        const float dl1 = p1 * (__uint_as_float(dp[e + 1]) - dr);
        dgain_acc = fmaf(dl0, bias[e], fmaf(dl1, bias[e + 1], dgain_acc));
        dtz_acc = fmaf(dl0, s0, fmaf(dl1, s1, dtz_acc));
        pk[e >> 1] = pack_bf16x2(dl0 * as, dl1 * as);
      }
      tmem_st16(tmem + lane_base + 64 * b + 32 * wg, pk);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&ds_full[b]);
    }
    if (ok && !*abort_flag) ok = warp_wait(o_final, 0, kErrWaitAttention);
    if (!ok) *abort_flag = 1;
    if (ok) {
      tc_fence_after();
#pragma unroll 1
      for (int c0 = wg * (D / 2); c0 < (wg + 1) * (D / 2); c0 += 32) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_base + Cfg::kColDQ + c0, o);
        tmem_ld_wait();
        if (row_ok) {
          float4* dst = reinterpret_cast<float4*>(p.dq + int64_t(grow) * p.hq * D + h * D + c0);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            dst[e] = make_float4(__uint_as_float(o[4 * e]), __uint_as_float(o[4 * e + 1]),
                                 __uint_as_float(o[4 * e + 2]), __uint_as_float(o[4 * e + 3]));
        }
      }
    }
    // dgain / dtemp of this (head, row block): fixed-order sums over lanes, then warps
    float vg = dgain_acc, vt = dtz_acc * ratio_r * p.sm_scale;
#pragma unroll
    for (int off = 16; off; off >>= 1) {
      vg += __shfl_xor_sync(0xffffffffu, vg, off);
      vt += __shfl_xor_sync(0xffffffffu, vt, off);
    }
    if (lane == 0) {
      red[2 * warp] = vg;
      red[2 * warp + 1] = vt;
    }
    asm volatile("bar.sync 1, 256;" ::: "memory");
    if (threadIdx.x == 0) {
      float sg = 0.0f, st = 0.0f;
      for (int w = 0; w < 8; ++w) {
        sg += red[2 * w];
        st += red[2 * w + 1];
      }
      p.dgt_part[(int64_t(h) * p.nkb + qb) * 2] = sg;
      p.dgt_part[(int64_t(h) * p.nkb + qb) * 2 + 1] = st;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    __syncwarp();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// dK, dV (and the dbias partials of the KV head)
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(kBwdTcThreads, 1)
    k_attn_bwd_kv_tc(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmDO,
                     const __grid_constant__ CUtensorMap tmPar, AttnBwdParams p) {
  using Cfg = BwdKvCfg<D>;
  constexpr int BR = Cfg::BR;
  constexpr int kDBoxes = D / 64;
  extern __shared__ uint8_t bwd_tc_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(bwd_tc_smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = smem;
  uint8_t* sV = smem + Cfg::kOffV;
  uint8_t* sQ = smem + Cfg::kOffQ;
  uint8_t* sDO = smem + Cfg::kOffDO;
  const float4* sPar = reinterpret_cast<const float4*>(smem + Cfg::kOffPar);  // [stage][64 rows] (a2, nl, D_r, as)
  float* red = reinterpret_cast<float*>(smem + Cfg::kOffRed);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kOffBars);
  constexpr int kS = Cfg::kStages;
  uint64_t* kv_full = bars + 0;       // the K and V blocks
  uint64_t* r_full = bars + 1;        // [kS] Q, dO tile n and its row constants (stage n % kS)
  uint64_t* mm_done = r_full + kS;    // [kS] dV, dK MMAs of tile n complete: stage n % kS free
  uint64_t* s_full = mm_done + kS;    // [2] S^T and dP^T of tile n in buffer n % 2
  uint64_t* p_full = s_full + 2;      // [2] P^T and dS^T of tile n written (256 arrivals)
  uint64_t* o_final = p_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(o_final + 1);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // longest first: key block 0 is seen by every row
  const int kb = static_cast<int>(blockIdx.x) / p.hkv;
  const int g = static_cast<int>(blockIdx.x) % p.hkv;
  const int key0 = kb * Cfg::BK;
  const int ntq = (p.m - key0 + BR - 1) / BR;  // row tiles per head
  const int nt = ntq * p.group;                // tile n: head g * group + n / ntq, rows key0 + 64 (n % ntq)

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < kS; ++s) {
      mbar_init(&r_full[s], 1);
      mbar_init(&mm_done[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], 256);
    }
    mbar_init(o_final, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmDO);
      prefetch_tmap(&tmPar);
      mbar_arrive_expect_tx(kv_full, 2 * Cfg::kKBytes);
      for (int b = 0; b < kDBoxes; ++b) {
        tma_load_2d(sK + b * Cfg::kKBlk, &tmK, kv_full, g * D + 64 * b, key0);
        tma_load_2d(sV + b * Cfg::kKBlk, &tmV, kv_full, g * D + 64 * b, key0);
      }
      for (int n = 0; n < nt; ++n) {
        const int s = n % kS;
        if (n >= kS && !mbar_wait(&mm_done[s], ((n - kS) / kS) & 1, kErrWaitAttention)) {
          *abort_flag = 1;
          break;
        }
        const int h = g * p.group + n / ntq;
        const int row0 = key0 + BR * (n % ntq);
        mbar_arrive_expect_tx(&r_full[s], 2 * Cfg::kRBytes + BR * 16);
        for (int b = 0; b < kDBoxes; ++b) {
          tma_load_2d(sQ + s * Cfg::kRBytes + b * Cfg::kRBlk, &tmQ, &r_full[s], h * D + 64 * b, row0);
          tma_load_2d(sDO + s * Cfg::kRBytes + b * Cfg::kRBlk, &tmDO, &r_full[s], h * D + 64 * b, row0);
        }
        tma_load_1d(const_cast<float4*>(sPar) + s * BR, &tmPar, &r_full[s],
                    static_cast<int32_t>((int64_t(h) * p.m_pad + row0) * 4));
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_t = idesc_bf16_f32(128, BR, false, false);
      constexpr uint32_t idesc_acc = idesc_bf16_f32(128, D, false, true);
      const uint64_t dk0 = sdesc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t dv0 = sdesc_sw128(smem_u32(sV), 16, 1024);
      const uint64_t dq0 = sdesc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t ddo0 = sdesc_sw128(smem_u32(sDO), 16, 1024);
      const uint64_t dqmn0 = sdesc_sw128(smem_u32(sQ), Cfg::kRBlk, 1024);
      const uint64_t ddomn0 = sdesc_sw128(smem_u32(sDO), Cfg::kRBlk, 1024);
      auto issue_s = [&](int n) {
        const int b = n & 1, s = n % kS;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ao = ((kk >> 2) * Cfg::kKBlk + (kk & 3) * 32) >> 4;
          const uint32_t bo = (s * Cfg::kRBytes + (kk >> 2) * Cfg::kRBlk + (kk & 3) * 32) >> 4;
          umma_ss(tmem + 64 * b, dk0 + ao, dq0 + bo, idesc_t, kk != 0 ? 1u : 0u);
          umma_ss(tmem + Cfg::kColDP + 64 * b, dv0 + ao, ddo0 + bo, idesc_t, kk != 0 ? 1u : 0u);
        }
        umma_commit(&s_full[b]);
      };
      auto issue_acc = [&](int n) {
        const int b = n & 1, s = n % kS;
#pragma unroll
        for (int kk = 0; kk < BR / 16; ++kk) {
          const uint64_t bo = (s * Cfg::kRBytes + kk * 16 * 128) >> 4;
          const uint32_t acc = (n | kk) != 0 ? 1u : 0u;
          umma_ts(tmem + Cfg::kColDV, tmem + 64 * b + bwd_packed_col(kk), ddomn0 + bo, idesc_acc, acc);
          umma_ts(tmem + Cfg::kColDK, tmem + Cfg::kColDP + 64 * b + bwd_packed_col(kk), dqmn0 + bo, idesc_acc, acc);
        }
        umma_commit(&mm_done[s]);
      };
      bool ok = mbar_wait2(kv_full, 0, &r_full[0], 0, kErrWaitAttention);
      if (ok) {
        tc_fence_after();
        issue_s(0);
      }
      if (ok && nt > 1 && (ok = mbar_wait(&r_full[1], 0, kErrWaitAttention))) {
        tc_fence_after();
        issue_s(1);
      }
      for (int n = 0; ok && n < nt; ++n) {
        const bool next = n + 2 < nt;
        ok = mbar_wait(&p_full[n & 1], (n >> 1) & 1, kErrWaitAttention) &&
             (!next || mbar_wait(&r_full[(n + 2) % kS], ((n + 2) / kS) & 1, kErrWaitAttention));
        if (!ok) break;
        tc_fence_after();
        issue_acc(n);
        if (next) issue_s(n + 2);  // into the buffers the accumulation of tile n has just read
      }
      if (ok) umma_commit(o_final);
      else *abort_flag = 1;
    }
  } else {
    // ------------------------------------------------------------ elementwise warpgroups
    const int wg = warp >> 2, q4 = warp & 3;
    const int kl = q4 * 32 + lane, key = key0 + kl;  // this thread's key
    const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
    const float bias_c = (p.bias && key < p.m) ? p.bias[key] : 0.0f;
    float dbias_acc = 0.0f;
    bool ok = true;
    for (int n = 0; n < nt; ++n) {
      const int b = n & 1, s = n % kS;
      const int h = g * p.group + n / ntq;
      const int i = n % ntq;
      bool rdy = !*abort_flag &&
                 mbar_wait2(&s_full[b], (n >> 1) & 1, &r_full[s], (n / kS) & 1, kErrWaitAttention);
      if (!__all_sync(0xffffffffu, rdy)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sr[32], dp[32];
      tmem_ld32(tmem + lane_base + 64 * b + 32 * wg, sr);
      tmem_ld32(tmem + lane_base + Cfg::kColDP + 64 * b + 32 * wg, dp);
      tmem_ld_wait();
      const float gain = p.gain[h];
      const float gb2 = gain * kLog2e * bias_c;
      const float4* par = sPar + s * BR + 32 * wg;
      const int r0 = key0 + BR * i + 32 * wg;  // row of column 0 of this half
      const bool diag = i < 2;                 // rows before key0 + 128 meet the causal mask
      uint32_t pp[16], pd[16];
#pragma unroll
      for (int e = 0; e < 32; e += 4) {
        float pv[4], dsv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float4 c = par[e + u];  // (a2, nl, D_r, as) of the row
          float x = fmaf(c.x, __uint_as_float(sr[e + u]), gb2 + c.y);
          if (diag && key > r0 + e + u) x = -INFINITY;
          pv[u] = ex2_approx(x);
          const float dl = pv[u] * (__uint_as_float(dp[e + u]) - c.z);
          dbias_acc = fmaf(gain, dl, dbias_acc);
          dsv[u] = dl * c.w;
        }
        pp[e >> 1] = pack_bf16x2(pv[0], pv[1]);
        pp[(e >> 1) + 1] = pack_bf16x2(pv[2], pv[3]);
        pd[e >> 1] = pack_bf16x2(dsv[0], dsv[1]);
        pd[(e >> 1) + 1] = pack_bf16x2(dsv[2], dsv[3]);
      }
      tmem_st16(tmem + lane_base + 64 * b + 32 * wg, pp);
      tmem_st16(tmem + lane_base + Cfg::kColDP + 64 * b + 32 * wg, pd);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_full[b]);
    }
    if (ok && !*abort_flag) ok = warp_wait(o_final, 0, kErrWaitAttention);
    if (!ok) *abort_flag = 1;
    if (ok) {
      // warpgroup 0 writes dV, warpgroup 1 dK (fp32 rows of this key)
      tc_fence_after();
      const uint32_t col = wg ? Cfg::kColDK : Cfg::kColDV;
      float* dst_row = (wg ? p.dk : p.dv) + int64_t(key) * p.hkv * D + g * D;
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_base + col + c0, o);
        tmem_ld_wait();
        if (key < p.m) {
          float4* dst = reinterpret_cast<float4*>(dst_row + c0);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            dst[e] = make_float4(__uint_as_float(o[4 * e]), __uint_as_float(o[4 * e + 1]),
                                 __uint_as_float(o[4 * e + 2]), __uint_as_float(o[4 * e + 3]));
        }
      }
    }
    // the two warpgroups each summed half of every tile's rows: add them in a fixed order
    if (wg == 1) red[kl] = dbias_acc;
    asm volatile("bar.sync 1, 256;" ::: "memory");
    if (wg == 0 && key < p.m) p.dbias_part[int64_t(g) * p.m + key] = dbias_acc + red[kl];
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    __syncwarp();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace tg

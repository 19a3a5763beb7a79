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
//   key tiles of 64 up to the diagonal.  Q and dO are copied once into tensor
//   memory, so S = Q K^T and dP = dO V^T are TS-MMAs (only K and V come from
//   shared memory) into double-buffered tensor memory; two warpgroups (one
//   thread per row, each taking 32 of a tile's 64 keys) turn them into dS,
//   written as bf16 pairs over the first 16 columns of their half of the S
//   buffer, and the MMA thread accumulates dQ += dS K as a TS-MMA (K MN-major
//   from shared memory).  The row's dgain / dtemp terms are summed on the way.
// k_attn_bwd_kv_tc: one CTA per (query head h, block of 128 keys), walking the
//   query tiles of 64 rows from the diagonal on.
//   S^T = K Q^T and dP^T = V dO^T (one thread per key), P^T and dS^T as bf16
//   pairs over their own columns, then dV += P^T dO and dK += dS^T Q as
//   TS-MMAs; both accumulators stay in tensor memory over the whole walk.  The
//   query heads that share a KV head add their (dV, dK) through the workspace
//   in head order (the last CTA of the group to finish does the sum).  The
//   per-row constants of a tile (from k_attn_bwd_prep) come by TMA into the
//   same stage as the Q / dO tiles.
// k_attn_bwd_prep: D_r and the per-row constants (a_r sm_scale log2 e,
//   -lse_r log2 e, -D_r, a_r sm_scale) of every head and row, interleaved by
//   row pairs so that the elementwise loops read them as packed f32x2 pairs;
//   rows past m masked (P = 0 there).  The elementwise arithmetic runs on
//   f32x2 pairs (fma/add/mul.rn.f32x2: per-lane IEEE results).
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
  // S[b] at 64 b, dP[b] at 128 + 64 b, dQ, then Q and dO as packed bf16 pairs (the A operands)
  static constexpr uint32_t kColDP = 128, kColDQ = 256, kColQ = 256 + D, kColDO = 256 + D + D / 2;
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

__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// ---------------------------------------------------------------------------
// Epilogue staging: a warp holds 32 rows (lane = row) x 32 fp32 columns from a
// tcgen05.ld; it writes them into a 4 KB swizzled area (16-byte chunk c of row
// r at c ^ (r & 7): no bank conflicts either way) and reads them back so that
// eight lanes cover one row's 128 contiguous bytes, four rows per instruction.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float4* stage_slot(float* stage, int row, int chunk) {
  return reinterpret_cast<float4*>(stage) + row * 8 + (chunk ^ (row & 7));
}

__device__ __forceinline__ void stage_rows32(float* stage, const uint32_t (&o)[32]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int c = 0; c < 8; ++c)
    *stage_slot(stage, lane, c) = make_float4(__uint_as_float(o[4 * c]), __uint_as_float(o[4 * c + 1]),
                                              __uint_as_float(o[4 * c + 2]), __uint_as_float(o[4 * c + 3]));
  __syncwarp();
}

// Coalesced write-out of a staged 32 x 32 block: row i goes to dst + (row0 + i) * ld, rows >= nrows skipped.
__device__ __forceinline__ void stage_store32(float* stage, float* dst, int64_t ld, int row0, int nrows) {
  const int lane = threadIdx.x & 31, cc = lane & 7;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int r = (lane >> 3) + 4 * k;
    if (row0 + r < nrows) reinterpret_cast<float4*>(dst + int64_t(row0 + r) * ld)[cc] = *stage_slot(stage, r, cc);
  }
  __syncwarp();  // the area is free for the next block
}

// ---------------------------------------------------------------------------
// Per-row constants: one warp per row, all heads (rows m .. m_pad - 1 masked).
// A 16-byte load per lane covers 256 / D heads (D / 8 lanes each); all loads
// of the row are issued before the lane-group reductions.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) k_attn_bwd_prep(AttnBwdParams p) {
  constexpr int kLanesPerHead = D / 8, kHeadsPerLoad = 32 / kLanesPerHead;
  const int r = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (r >= p.m_pad) return;  // warp-uniform
  // rows r and r ^ 1 share 8 floats per head: (a2, a2', nl, nl', -D, -D', as, as')
  auto dst = [&](int h) { return p.rowpar + (int64_t(h) * (p.m_pad / 2) + r / 2) * 8 + (r & 1); };
  if (r >= p.m) {
    for (int h = lane; h < p.hq; h += 32) {
      float* d = dst(h);
      d[0] = 0.0f;
      d[2] = -INFINITY;
      d[4] = 0.0f;
      d[6] = 0.0f;
    }
    return;
  }
  const float ratio_r = p.ratio ? p.ratio[r] : 1.0f;
  const uint4* go = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.dout) + int64_t(r) * p.lddo);
  const uint4* oo = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.o) + int64_t(r) * p.ldo);
  const int sub = lane % kLanesPerHead;
  const int niter = (p.hq + kHeadsPerLoad - 1) / kHeadsPerLoad;
  // chunks of kChunk loads per operand, all issued before any use (the stores
  // of a chunk would otherwise keep the next chunk's loads behind them)
  constexpr int kChunk = 8;
  for (int it0 = 0; it0 < niter; it0 += kChunk) {
    uint4 a[kChunk], b[kChunk];
    float lse[kChunk], th[kChunk];
#pragma unroll
    for (int c = 0; c < kChunk; ++c) {
      const int h = (it0 + c) * kHeadsPerLoad + lane / kLanesPerHead;
      const bool hv = it0 + c < niter && h < p.hq;
      a[c] = hv ? go[h * kLanesPerHead + sub] : make_uint4(0, 0, 0, 0);           // dO: read again by the MMAs
      b[c] = hv ? __ldcs(oo + h * kLanesPerHead + sub) : make_uint4(0, 0, 0, 0);  // o: this pass only
      lse[c] = (hv && sub == 0) ? p.lse[int64_t(h) * p.m + r] : 0.0f;
      th[c] = (hv && sub == 0) ? p.temp[h] : 0.0f;
    }
#pragma unroll
    for (int c = 0; c < kChunk; ++c) {
      const int h = (it0 + c) * kHeadsPerLoad + lane / kLanesPerHead;
      const bool hv = it0 + c < niter && h < p.hq;
      float sdot = bf16_lo(a[c].x) * bf16_lo(b[c].x) + bf16_hi(a[c].x) * bf16_hi(b[c].x) +
                   bf16_lo(a[c].y) * bf16_lo(b[c].y) + bf16_hi(a[c].y) * bf16_hi(b[c].y) +
                   bf16_lo(a[c].z) * bf16_lo(b[c].z) + bf16_hi(a[c].z) * bf16_hi(b[c].z) +
                   bf16_lo(a[c].w) * bf16_lo(b[c].w) + bf16_hi(a[c].w) * bf16_hi(b[c].w);
#pragma unroll
      for (int off = kLanesPerHead / 2; off; off >>= 1) sdot += __shfl_xor_sync(0xffffffffu, sdot, off);
      if (hv && sub == 0) {
        const float as = th[c] * ratio_r * p.sm_scale;
        float* d = dst(h);
        d[0] = as * kLog2e;
        d[2] = -lse[c] * kLog2e;
        d[4] = -sdot;
        d[6] = as;
      }
    }
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
  uint64_t* qt_ready = o_final + 1;    // Q and dO copied into tensor memory (256 arrivals)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(qt_ready + 1);
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
    mbar_init(qt_ready, 256);
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
      const uint64_t dk0 = sdesc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t dv0 = sdesc_sw128(smem_u32(sV), 16, 1024);
      const uint64_t dkmn0 = sdesc_sw128(smem_u32(sK), Cfg::kKVBlk, 1024);
      // S = Q K^T and dP = dO V^T take Q and dO from tensor memory (TS): per
      // MMA only the 64-key K or V slice is read from shared memory
      auto issue_s = [&](int j) {
        const int b = j & 1, s = j % kS;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t bo = (s * Cfg::kKVBytes + (kk >> 2) * Cfg::kKVBlk + (kk & 3) * 32) >> 4;
          umma_ts(tmem + 64 * b, tmem + Cfg::kColQ + kk * 8, dk0 + bo, idesc_s, kk != 0 ? 1u : 0u);
          umma_ts(tmem + Cfg::kColDP + 64 * b, tmem + Cfg::kColDO + kk * 8, dv0 + bo, idesc_s, kk != 0 ? 1u : 0u);
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
      bool ok = mbar_wait2(qt_ready, 0, &kv_full[0], 0, kErrWaitAttention);
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
        // both barriers tested at once (each test holds back the next MMA issue for a round trip)
        const bool r0 = mbar_try_wait(smem_u32(&ds_full[j & 1]), (j >> 1) & 1);
        const bool r1 = !next || mbar_try_wait(smem_u32(&kv_full[(j + 2) % kS]), ((j + 2) / kS) & 1);
        if (!(r0 && r1))
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
    const float* pr = p.rowpar + (int64_t(h) * (p.m_pad / 2) + grow / 2) * 8 + (grow & 1);  // masked past m
    const float a2 = pr[0], nl = pr[2], ndr = pr[4], as = pr[6];
    const float gg = p.gain[h] * kLog2e;
    const uint64_t a2p = f2_pack(a2, a2), nlp = f2_pack(nl, nl), ndrp = f2_pack(ndr, ndr), asp = f2_pack(as, as),
                   ggp = f2_pack(gg, gg);
    uint64_t dgain2 = 0, dtz2 = 0;  // (even keys, odd keys) partial sums
    bool ok = true;
    // warpgroup 0 copies the Q rows, warpgroup 1 the dO rows, from their TMA
    // tiles (128-byte swizzled boxes of 64 columns) into tensor memory as
    // packed bf16 pairs: thread = row = TMEM lane
    if (warp_wait(q_full, 0, kErrWaitAttention)) {
      const uint8_t* tile = (wg ? sDO : sQ) + row * 128;
      const uint32_t col = wg ? Cfg::kColDO : Cfg::kColQ;
#pragma unroll
      for (int bx = 0; bx < kDBoxes; ++bx) {
        uint32_t v[32];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 x = *reinterpret_cast<const uint4*>(tile + bx * Cfg::kQBlk + ((c ^ (row & 7)) << 4));
          v[4 * c] = x.x;
          v[4 * c + 1] = x.y;
          v[4 * c + 2] = x.z;
          v[4 * c + 3] = x.w;
        }
        tmem_st32(tmem + lane_base + col + 32 * bx, v);
      }
      tmem_st_wait();
    } else {
      ok = false;
    }
    tc_fence_before();
    mbar_arrive(qt_ready);
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
      const uint64_t* bias2 = reinterpret_cast<const uint64_t*>(sBias + (j % kS) * BN + 32 * wg);
      const int key0 = j * BN + 32 * wg;
      const bool diag = key0 + 31 > qb * 128;  // warp-uniform
      uint32_t pk[16];
#pragma unroll
      for (int e = 0; e < 32; e += 2) {
        const uint64_t s2 = f2_pack(__uint_as_float(sr[e]), __uint_as_float(sr[e + 1]));
        const uint64_t b2 = bias2[e >> 1];
        float x0, x1;
        f2_unpack(f2_fma(a2p, s2, f2_fma(ggp, b2, nlp)), x0, x1);
        if (diag) {
          if (key0 + e > grow) x0 = -INFINITY;
          if (key0 + e + 1 > grow) x1 = -INFINITY;
        }
        const uint64_t p2 = f2_pack(ex2_approx(x0), ex2_approx(x1));
        const uint64_t dl2 = f2_mul(p2, f2_add(f2_pack(__uint_as_float(dp[e]), __uint_as_float(dp[e + 1])), ndrp));
        dgain2 = f2_fma(dl2, b2, dgain2);
        dtz2 = f2_fma(dl2, s2, dtz2);
        float d0, d1;
        f2_unpack(f2_mul(dl2, asp), d0, d1);
        pk[e >> 1] = pack_bf16x2(d0, d1);
      }
      tmem_st16(tmem + lane_base + 64 * b + 32 * wg, pk);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&ds_full[b]);
    }
    if (ok && !*abort_flag) ok = warp_wait(o_final, 0, kErrWaitAttention);
    if (!ok) *abort_flag = 1;
    if (ok) {
      // dQ through a per-warp staging area in the (now idle) K ring
      tc_fence_after();
      float* stage = reinterpret_cast<float*>(sK) + warp * 1024;
#pragma unroll 1
      for (int c0 = wg * (D / 2); c0 < (wg + 1) * (D / 2); c0 += 32) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_base + Cfg::kColDQ + c0, o);
        tmem_ld_wait();
        stage_rows32(stage, o);
        stage_store32(stage, p.dq + h * D + c0, int64_t(p.hq) * D, qb * 128 + q4 * 32, p.m);
      }
    }
    // dgain / dtemp of this (head, row block): fixed-order sums over lanes, then warps
    float g0, g1, t0, t1;
    f2_unpack(dgain2, g0, g1);
    f2_unpack(dtz2, t0, t1);
    float vg = g0 + g1, vt = (t0 + t1) * ratio_r * p.sm_scale;
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
  const float4* sPar = reinterpret_cast<const float4*>(smem + Cfg::kOffPar);  // [stage][32 row pairs][2] float4
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
  const int kb = static_cast<int>(blockIdx.x) / p.hq;
  const int h = static_cast<int>(blockIdx.x) % p.hq;
  const int g = h / p.group, u = h % p.group;
  const int key0 = kb * Cfg::BK;
  const int nt = (p.m - key0 + BR - 1) / BR;  // row tiles: rows key0 + 64 n

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
        const int row0 = key0 + BR * n;
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
        const bool r0 = mbar_try_wait(smem_u32(&p_full[n & 1]), (n >> 1) & 1);
        const bool r1 = !next || mbar_try_wait(smem_u32(&r_full[(n + 2) % kS]), ((n + 2) / kS) & 1);
        if (!(r0 && r1))
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
    const float gain = p.gain[h];
    const float gb2 = gain * kLog2e * bias_c;
    const uint64_t gb2p = f2_pack(gb2, gb2), gainp = f2_pack(gain, gain);
    uint64_t dbias2 = 0;  // (even rows, odd rows) partial sums
    bool ok = true;
    for (int n = 0; n < nt; ++n) {
      const int b = n & 1, s = n % kS;
      const int i = n;
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
      // (a2, a2', nl, nl') and (-D, -D', as, as') of each row pair of this half
      const float4* par = sPar + s * BR + 32 * wg;
      const int r0 = key0 + BR * i + 32 * wg;  // row of column 0 of this half
      const bool diag = i < 2;                 // rows before key0 + 128 meet the causal mask
      uint32_t pp[16], pd[16];
#pragma unroll
      for (int e = 0; e < 32; e += 2) {
        const float4 c0 = par[e], c1 = par[e + 1];
        const uint64_t s2 = f2_pack(__uint_as_float(sr[e]), __uint_as_float(sr[e + 1]));
        float x0, x1;
        f2_unpack(f2_fma(f2_pack(c0.x, c0.y), s2, f2_add(gb2p, f2_pack(c0.z, c0.w))), x0, x1);
        if (diag) {
          if (key > r0 + e) x0 = -INFINITY;
          if (key > r0 + e + 1) x1 = -INFINITY;
        }
        const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
        const uint64_t dl2 = f2_mul(f2_pack(p0, p1), f2_add(f2_pack(__uint_as_float(dp[e]), __uint_as_float(dp[e + 1])),
                                                            f2_pack(c1.x, c1.y)));
        dbias2 = f2_fma(gainp, dl2, dbias2);
        float d0, d1;
        f2_unpack(f2_mul(dl2, f2_pack(c1.z, c1.w)), d0, d1);
        pp[e >> 1] = pack_bf16x2(p0, p1);
        pd[e >> 1] = pack_bf16x2(d0, d1);
      }
      tmem_st16(tmem + lane_base + 64 * b + 32 * wg, pp);
      tmem_st16(tmem + lane_base + Cfg::kColDP + 64 * b + 32 * wg, pd);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_full[b]);
    }
    if (ok && !*abort_flag) ok = warp_wait(o_final, 0, kErrWaitAttention);
    if (!ok) *abort_flag = 1;
    // the two warpgroups each summed half of every tile's rows: add them in a fixed order
    float dbl, dbh;
    f2_unpack(dbias2, dbl, dbh);
    const float dbias_acc = dbl + dbh;
    if (wg == 1) red[kl] = dbias_acc;
    asm volatile("bar.sync 1, 256;" ::: "memory");
    if (wg == 0 && key < p.m) p.dbias_part[int64_t(h) * p.m + key] = dbias_acc + red[kl];
    const bool good = !*abort_flag;  // agreed by every elementwise thread (read after the barrier)
    // (dV, dK) of this head: warpgroup 0 holds the dV columns, warpgroup 1 the dK columns.
    // With GQA the heads of the group meet here: every CTA but the last (by ticket)
    // publishes its partial; the last adds all heads' partials in head order.
    const uint32_t col = wg ? Cfg::kColDK : Cfg::kColDV;
    float* dst_base = (wg ? p.dk : p.dv) + g * D;  // row 0 of this KV head's columns
    const int nslots = p.hkv * (p.m_pad / Cfg::BK);
    const int slot = g * (p.m_pad / Cfg::BK) + kb;
    int role = 0;  // 0: write the result directly, 1: publish a partial, 2: merge the partials
    if (good && p.group > 1) {
      if (threadIdx.x == 0) tmem_slot[2] = atomicAdd(&p.kv_ctr[slot], 1u) == unsigned(p.group - 1) ? 2u : 1u;
      asm volatile("bar.sync 1, 256;" ::: "memory");
      role = static_cast<int>(tmem_slot[2]);
    }
    float* part = p.kv_part + (int64_t(slot) * p.group) * Cfg::BK * 2 * D;  // [group][128][2 D]
    // per-warp staging area in the (now idle) Q ring
    float* stage = reinterpret_cast<float*>(sQ) + warp * 1024;
    if (good && role == 1) {
      tc_fence_after();
      float* mine = part + int64_t(u) * Cfg::BK * 2 * D + (wg ? D : 0);
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_base + col + c0, o);
        tmem_ld_wait();
        stage_rows32(stage, o);
        stage_store32(stage, mine + c0, 2 * D, q4 * 32, Cfg::BK);
      }
      __threadfence();
      asm volatile("bar.sync 1, 256;" ::: "memory");
      if (threadIdx.x == 0) atomicAdd(&p.kv_ctr[nslots + slot], 1u);
    }
    bool merge_ok = true;
    if (good && role == 2) {
      // the other heads' CTAs took their tickets before this one, so they are
      // running; wait (bounded) until all have published
      if (threadIdx.x == 0) {
        const uint64_t t0 = globaltimer_ns();
        uint32_t okw = 1;
        while (ld_acquire_gpu(&p.kv_ctr[nslots + slot]) < unsigned(p.group - 1)) {
          if (globaltimer_ns() - t0 > kWaitLimitNs) {
            raise_error(kErrWaitAttention, 2);
            okw = 0;
            break;
          }
        }
        tmem_slot[3] = okw;
      }
      asm volatile("bar.sync 1, 256;" ::: "memory");
      merge_ok = tmem_slot[3] != 0;
    }
    if (good && role != 1 && merge_ok) {
      tc_fence_after();
      const int cc = lane & 7;
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_base + col + c0, o);
        tmem_ld_wait();
        stage_rows32(stage, o);
        if (role == 2) {
          // sum over the group's heads in head order, on the staged (coalesced)
          // layout; the eight rows of a head are fetched together
          float4 acc[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) acc[k] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
          for (int w = 0; w < p.group; ++w) {
            float4 x[8];
            if (w == u) {
#pragma unroll
              for (int k = 0; k < 8; ++k) x[k] = *stage_slot(stage, (lane >> 3) + 4 * k, cc);
            } else {
              const float4* src = reinterpret_cast<const float4*>(part + (int64_t(w) * Cfg::BK + q4 * 32) * 2 * D +
                                                                  (wg ? D : 0) + c0) + cc;
#pragma unroll
              for (int k = 0; k < 8; ++k) x[k] = __ldcg(src + ((lane >> 3) + 4 * k) * (2 * D / 4));
            }
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              acc[k].x += x[k].x;
              acc[k].y += x[k].y;
              acc[k].z += x[k].z;
              acc[k].w += x[k].w;
            }
          }
#pragma unroll
          for (int k = 0; k < 8; ++k) *stage_slot(stage, (lane >> 3) + 4 * k, cc) = acc[k];
          __syncwarp();
        }
        stage_store32(stage, dst_base + c0, int64_t(p.hkv) * D, key0 + q4 * 32, p.m);
      }
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

}  // namespace tg

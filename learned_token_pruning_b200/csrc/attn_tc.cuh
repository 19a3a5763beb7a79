// Token-gated causal GQA flash attention on the 5th-generation tensor cores.
//
// Method ("TokenGate and T2Quant: a close reading", §4.1 token-gated
// attention, head-wise gain, temperature scaling): for query head h, KV head g
// and kept rows c <= r
//     l_rc = temp_h * ratio_r * sm_scale * (q_r . k_c) + gain_h * bias_c
//     o_r  = sum_c softmax_c(l_r.) v_c
// computed in base 2: x = a_r * S_rc + beta_c with a_r = temp_h * ratio_r *
// sm_scale * log2(e) (one scale per row) and beta_c = gain_h * log2(e) * bias_c
// (one offset per key).
//
// One CTA owns a 128-row query block of TWO query heads that share a KV head
// (GQA), so every K/V tile fetched by TMA feeds two 128x128 score tiles.
//   warps 0-3  softmax warpgroup 0 (query tile 0), one thread per row
//   warps 4-7  softmax warpgroup 1 (query tile 1)
//   warp 8     TMA producer (Q once, then K and V tiles through a 2-stage ring)
//   warp 9     TMEM allocator and single-thread tcgen05.mma issuer
// Tensor memory (512 columns): S0 [0,128), S1 [128,256), O0 and O1 after them.
// S_i = Q_i K^T is an SS-MMA (both operands in shared memory, K-major); the
// softmax warps read S_i with tcgen05.ld, write P_i = exp2(x - m) as packed
// bf16 over the first 64 columns of S_i, and O_i += P_i V is a TS-MMA with P
// taken from tensor memory and V (MN-major) from shared memory.  The running
// row maximum is only moved when it grows by more than 8 (log2 units), and O is
// then rescaled in tensor memory by the softmax warps themselves; P <= 2^8 in
// between, which bf16 and the fp32 accumulators hold exactly enough.
// Every MMA is issued by one thread, so tcgen05 executes them in issue order:
// QK_i(j+1), which overwrites S_i, is issued after PV_i(j), which reads P_i
// from the same columns, and the commit after QK_i(j+1) also covers PV_i(j),
// which is what lets the softmax warps touch O_i after waiting on it.
#pragma once

#include "common.cuh"
#include "simt.cuh"

namespace tg {

constexpr int kAttnThreads = 320;

template <int D>
struct AttnCfg {
  static constexpr int BM = 128, BN = 128;
  static constexpr int kQBytes = BM * D * 2;   // one query tile
  static constexpr int kKVBytes = BN * D * 2;  // one K or V tile
  static constexpr int kBlk = 128 * 128;       // bytes of one 64-column TMA box of 128 rows
  static constexpr int kStages = 2;
  static constexpr int kColS0 = 0, kColS1 = 128, kColO0 = 256, kColO1 = 256 + D;
  // Data, barriers and bias tiles; D = 64 is padded so that only one CTA fits
  // on an SM and its 512-column TMEM allocation never waits on a neighbour.
  static constexpr size_t kSmemData = 2 * kQBytes + kStages * 2 * kKVBytes;
  static constexpr size_t kSmem = 1024 + (kSmemData < 120 * 1024 ? 120 * 1024 : kSmemData) + 2048 + 256;
};

struct AttnTcParams {
  int m, hq, hkv, group;
  int num_qtiles;
  const float* bias;
  const float* gain;
  const float* temp;
  const float* ratio;
  float scale_log2;  // sm_scale * log2(e)
  __nv_bfloat16* out;
  int64_t ldo;
  float* lse;
};

template <int D>
__global__ void __launch_bounds__(kAttnThreads, 1)
    k_attn_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, AttnTcParams p) {
  using Cfg = AttnCfg<D>;
  constexpr int kDBoxes = D / 64;
  extern __shared__ uint8_t attn_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(attn_smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                                    // [2][kQBytes]
  uint8_t* sK = sQ + 2 * Cfg::kQBytes;                   // [stages][kKVBytes]
  uint8_t* sV = sK + Cfg::kStages * Cfg::kKVBytes;       // [stages][kKVBytes]
  float* sBeta = reinterpret_cast<float*>(smem + (Cfg::kSmem - 1024 - 2048 - 256));  // [2 wg][2 buf][128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sBeta + 512);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;      // [2]
  uint64_t* v_full = bars + 3;      // [2]
  uint64_t* kv_empty = bars + 5;    // [2]
  uint64_t* s_full = bars + 7;      // [2]
  uint64_t* p_full = bars + 9;      // [2]
  uint64_t* o_final = bars + 11;
  uint64_t* beta_bar = bars + 12;   // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 14);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // longest query blocks first: the last row block has the most causal work
  const int pairs_per_kv = p.group / 2;
  const int per_tile = p.hkv * pairs_per_kv;
  const int t = p.num_qtiles - 1 - static_cast<int>(blockIdx.x) / per_tile;
  const int pair = static_cast<int>(blockIdx.x) % per_tile;
  const int g = pair / pairs_per_kv;
  const int h0 = g * p.group + 2 * (pair % pairs_per_kv);
  const int nt = t + 1;  // causal: key tiles 0..t

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&kv_empty[s], 1);
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], 128);
      mbar_init(&beta_bar[s], 128);
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
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      mbar_arrive_expect_tx(q_full, 2 * Cfg::kQBytes);
      for (int i = 0; i < 2; ++i)
        for (int b = 0; b < kDBoxes; ++b)
          tma_load_2d(sQ + i * Cfg::kQBytes + b * Cfg::kBlk, &tmQ, q_full, (h0 + i) * D + 64 * b, t * 128);
      for (int j = 0; j < nt; ++j) {
        const int s = j & 1;
        if (*abort_flag || !mbar_wait(&kv_empty[s], ((j >> 1) & 1) ^ 1, kErrWaitAttention)) {
          *abort_flag = 1;
          break;
        }
        mbar_arrive_expect_tx(&k_full[s], Cfg::kKVBytes);
        for (int b = 0; b < kDBoxes; ++b)
          tma_load_2d(sK + s * Cfg::kKVBytes + b * Cfg::kBlk, &tmK, &k_full[s], g * D + 64 * b, j * 128);
        mbar_arrive_expect_tx(&v_full[s], Cfg::kKVBytes);
        for (int b = 0; b < kDBoxes; ++b)
          tma_load_2d(sV + s * Cfg::kKVBytes + b * Cfg::kBlk, &tmV, &v_full[s], g * D + 64 * b, j * 128);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, false, true);
      auto issue_qk = [&](int i, int s) {
        const uint32_t qa = smem_u32(sQ + i * Cfg::kQBytes), kb = smem_u32(sK + s * Cfg::kKVBytes);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * Cfg::kBlk + (kk & 3) * 32;
          umma_ss(tmem + (i ? Cfg::kColS1 : Cfg::kColS0), sdesc_sw128(qa + off, 16, 1024),
                  sdesc_sw128(kb + off, 16, 1024), idesc_qk, kk != 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int i, int s, int j) {
        const uint32_t vb = smem_u32(sV + s * Cfg::kKVBytes);
#pragma unroll
        for (int kk = 0; kk < 128 / 16; ++kk) {
          umma_ts(tmem + (i ? Cfg::kColO1 : Cfg::kColO0), tmem + (i ? Cfg::kColS1 : Cfg::kColS0) + kk * 8,
                  sdesc_sw128(vb + kk * 16 * 128, Cfg::kBlk, 1024), idesc_pv, (j | kk) != 0 ? 1u : 0u);
        }
      };
      bool ok = mbar_wait(q_full, 0, kErrWaitAttention) && mbar_wait(&k_full[0], 0, kErrWaitAttention);
      if (ok) {
        tc_fence_after();
        issue_qk(0, 0);
        umma_commit(&s_full[0]);
        issue_qk(1, 0);
        umma_commit(&s_full[1]);
      }
      for (int j = 0; ok && j < nt; ++j) {
        const int s = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        ok = !*abort_flag && mbar_wait(&v_full[s], ph, kErrWaitAttention) &&
             mbar_wait(&p_full[0], j & 1, kErrWaitAttention);
        if (!ok) break;
        tc_fence_after();
        issue_pv(0, s, j);
        if (j + 1 < nt) {
          ok = mbar_wait(&k_full[s ^ 1], ((j + 1) >> 1) & 1, kErrWaitAttention);
          if (!ok) break;
          tc_fence_after();
          issue_qk(0, s ^ 1);
          umma_commit(&s_full[0]);
        }
        ok = mbar_wait(&p_full[1], j & 1, kErrWaitAttention);
        if (!ok) break;
        tc_fence_after();
        issue_pv(1, s, j);
        umma_commit(&kv_empty[s]);
        if (j + 1 < nt) {
          issue_qk(1, s ^ 1);
          umma_commit(&s_full[1]);
        }
      }
      if (ok) umma_commit(o_final);
      else *abort_flag = 1;
    }
  } else {
    // ------------------------------------------------------------ softmax warpgroups
    const int wg = warp >> 2;           // 0 or 1: which query tile
    const int q4 = warp & 3;            // TMEM lane quarter
    const int row = q4 * 32 + lane;     // row inside the query tile
    const int grow = t * 128 + row;
    const int h = h0 + wg;
    const int wtid = threadIdx.x & 127;
    const uint32_t colS = wg ? Cfg::kColS1 : Cfg::kColS0;
    const uint32_t colO = wg ? Cfg::kColO1 : Cfg::kColO0;
    const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
    const float a_row = grow < p.m ? p.temp[h] * (p.ratio ? p.ratio[grow] : 1.0f) * p.scale_log2 : 0.0f;
    const float gb = p.gain[h] * kLog2e;
    float* beta_wg = sBeta + wg * 256;
    float m_run = -INFINITY, l_run = 0.0f;
    bool ok = true;

    for (int j = 0; j < nt; ++j) {
      // this tile's key offsets: one per thread, exchanged through shared memory
      {
        const int c = j * 128 + wtid;
        beta_wg[(j & 1) * 128 + wtid] = (p.bias && c < p.m) ? gb * p.bias[c] : 0.0f;
        mbar_arrive(&beta_bar[wg]);
      }
      if (*abort_flag || !warp_wait(&beta_bar[wg], j & 1, kErrWaitAttention) ||
          !warp_wait(&s_full[wg], j & 1, kErrWaitAttention)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float* beta = beta_wg + (j & 1) * 128;
      uint32_t s0[32], s1[32], s2[32], s3[32];
      tmem_ld32(tmem + lane_base + colS + 0, s0);
      tmem_ld32(tmem + lane_base + colS + 32, s1);
      tmem_ld32(tmem + lane_base + colS + 64, s2);
      tmem_ld32(tmem + lane_base + colS + 96, s3);
      tmem_ld_wait();
      const bool diag = (j == t);
      float mx = -INFINITY;
      auto logits = [&](uint32_t(&r)[32], int c0) {
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const float4 b4 = *reinterpret_cast<const float4*>(beta + c0 + e);
          const float bb[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            float x = fmaf(a_row, __uint_as_float(r[e + u]), bb[u]);
            if (diag && c0 + e + u > row) x = -INFINITY;
            r[e + u] = __float_as_uint(x);
            mx = fmaxf(mx, x);
          }
        }
      };
      logits(s0, 0);
      logits(s1, 32);
      logits(s2, 64);
      logits(s3, 96);
      // lazy rescaling: the reference maximum only moves when the row maximum
      // exceeds it by more than 8 (so every p stays <= 2^8)
      // (per row: the branch below is divergent, so it holds no warp-collective op)
      float sc = 1.0f;
      if (mx > m_run + 8.0f) {
        if (j > 0) sc = exp2f(m_run - mx);
        m_run = mx;
      }
      float sum = 0.0f;
      auto emit_p = [&](const uint32_t(&r)[32], int c0) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float p0 = exp2f(__uint_as_float(r[2 * e]) - m_run);
          const float p1 = exp2f(__uint_as_float(r[2 * e + 1]) - m_run);
          sum += p0 + p1;
          pk[e] = pack_bf16x2(p0, p1);
        }
        // P overwrites the first 64 columns of S as packed bf16 pairs
        tmem_st16(tmem + lane_base + colS + c0 / 2, pk);
      };
      emit_p(s0, 0);
      emit_p(s1, 32);
      emit_p(s2, 64);
      emit_p(s3, 96);
      l_run = l_run * sc + sum;
      // tcgen05.ld/st are warp-collective (.sync.aligned): the whole warp
      // rescales its 32 rows if any of them needs it, the others with sc = 1
      if (__any_sync(0xffffffffu, sc != 1.0f)) {
        // O_i holds the sum over earlier tiles (its last PV finished before
        // s_full fired) and no PV into it is issued before p_full below
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_base + colO + c0, o);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * sc);
          tmem_st32(tmem + lane_base + colO + c0, o);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_full[wg]);
    }
    if (ok && !*abort_flag) ok = warp_wait(o_final, 0, kErrWaitAttention);
    if (ok) {
      tc_fence_after();
      const float inv = 1.0f / l_run;
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_base + colO + c0, o);
        tmem_ld_wait();
        if (grow < p.m) {
          uint4* dst = reinterpret_cast<uint4*>(p.out + static_cast<int64_t>(grow) * p.ldo + h * D + c0);
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(o[8 * v + 0]) * inv, __uint_as_float(o[8 * v + 1]) * inv);
            w.y = pack_bf16x2(__uint_as_float(o[8 * v + 2]) * inv, __uint_as_float(o[8 * v + 3]) * inv);
            w.z = pack_bf16x2(__uint_as_float(o[8 * v + 4]) * inv, __uint_as_float(o[8 * v + 5]) * inv);
            w.w = pack_bf16x2(__uint_as_float(o[8 * v + 6]) * inv, __uint_as_float(o[8 * v + 7]) * inv);
            dst[v] = w;
          }
        }
      }
      if (p.lse && grow < p.m) p.lse[static_cast<int64_t>(h) * p.m + grow] = (m_run + log2f(l_run)) * kLn2;
    } else {
      *abort_flag = 1;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    __syncwarp();  // the .sync.aligned dealloc needs the whole warp converged
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace tg

// Token-gated causal GQA flash attention on the 5th-generation tensor cores.
//
// Method ("TokenGate and T2Quant: a close reading", §4.1 token-gated
// attention, head-wise gain, temperature scaling): for query head h, KV head g
// and kept rows c <= r
//     l_rc = temp_h * ratio_r * sm_scale * (q_r . k_c) + gain_h * bias_c
//     o_r  = sum_c softmax_c(l_r.) v_c
// computed in base 2 with the head gain factored out of the row:
//     x_rc = g_h * y_rc,   y_rc = (a_r / g_h) * S_rc + bias_c,
//     a_r = temp_h * ratio_r * sm_scale * log2(e),  g_h = gain_h * log2(e),
// so the raw per-key bias tile, which TMA brings in with each K tile, serves
// both query heads of the CTA unchanged; the softmax runs on y (max, then
// exp2(g_h * (y - max))).
//
// One CTA owns a 128-row query block of TWO query heads that share a KV head
// (GQA), so every K/V tile fetched by TMA feeds two score tiles.  Keys come in
// tiles of 64.
//   warps 0-3  softmax warpgroup 0 (query head 0), one thread per row
//   warps 4-7  softmax warpgroup 1 (query head 1)
//   warp 8     TMA producer (Q once, then K + bias tiles through a 3-stage
//              ring and V tiles through a 2-stage ring)
//   warp 9     TMEM allocator and single-thread tcgen05.mma issuer
// Tensor memory (512 columns): S of each head double-buffered, 4 x 64 columns,
// then O0 and O1 (D columns each).  S = Q K^T is an SS-MMA into TMEM; the
// softmax reads S with tcgen05.ld and writes P = exp2(x - m) as bf16 pairs
// back over the first 32 columns of the same S buffer; O += P V is a TS-MMA
// (P from tensor memory, V MN-major from shared memory), which leaves the
// shared-memory port to Q, K and V.  Per key tile j the MMA thread issues
// P V of tile j for both heads and then Q K^T of tile j + 2 into the S
// buffers tile j used (in issue order, after P V has read P), so the scores
// of the next tile are ready when a softmax finishes and the loop is bounded
// by the slower of the softmax and the tensor core, not by their sum.
//
// The MMA thread checks the four barriers a tile needs (V, the P of both
// heads, K of tile j + 2) at once: each mbarrier check holds back its next
// tcgen05.mma for a shared-memory round trip while the tensor core's short
// queue drains.  The softmax does its elementwise arithmetic on packed pairs
// (fma/add.f32x2, three-input max), which halves its FMA-pipe instructions and
// leaves issue slots to the MMA thread.  The running row maximum only moves
// when it grows by more than 8 (log2 units); O is then rescaled in tensor
// memory by the softmax warps after the previous P V into it has completed.
#pragma once

#include "common.cuh"
#include "simt.cuh"

namespace tg {

constexpr int kAttnThreads = 320;
constexpr bool kPolyShare = false;  // evaluate a quarter of the exponentials with exp2_poly

template <int D>
struct AttnCfg {
  static constexpr int BM = 128, BN = 64;
  static constexpr int kQBytes = BM * D * 2;     // one query tile
  static constexpr int kKVBytes = BN * D * 2;    // one K or V tile
  static constexpr int kQBlk = BM * 128;         // one 64-column TMA box of a Q tile
  static constexpr int kKVBlk = BN * 128;        // one 64-column TMA box of a K or V tile
  static constexpr int kPBytes = BM * BN * 2;    // one P tile (128 rows x 64 keys, bf16)
  static constexpr int kKStages = 3, kVStages = 2;
  static constexpr int kColO0 = 256, kColO1 = 256 + D;
  static constexpr size_t kOffK = 2 * kQBytes;
  static constexpr size_t kOffV = kOffK + kKStages * kKVBytes;
  static constexpr size_t kOffP = kOffV + kVStages * kKVBytes;
  static constexpr size_t kOffBias = kOffP;  // (P lives in tensor memory, over its S columns)
  static constexpr size_t kOffBars = kOffBias + kKStages * BN * 4;  // 16 barriers + TMEM slot
  static constexpr size_t kData = kOffBars + 256;
  // D = 64 is padded so that only one CTA fits on an SM and its 512-column
  // TMEM allocation never waits on a neighbour
  static constexpr size_t kSmem = 1024 + (kData < 120 * 1024 ? 120 * 1024 : kData);
};

// TMEM column of head h's S buffer b
__device__ __forceinline__ uint32_t attn_col_s(int h, int b) { return static_cast<uint32_t>((h * 2 + b) * 64); }

struct AttnTcParams {
  int m, hq, hkv, group;
  int has_bias;
  int num_qtiles;
  const float* bias;
  const float* gain;
  const float* temp;
  const float* ratio;
  float scale_log2;  // sm_scale * log2(e)
  __nv_bfloat16* out;
  int64_t ldo;
  float* lse;
  // Key-range split of the longest query blocks (see AttnWork): query blocks
  // t >= ts run as two CTAs each; their partial results meet in `part`.
  int use_table;  // blocks take their work item from AttnWork (else: block b -> query block T-1-b/per_tile, whole)
  int ts;
  float4* part;   // [slot][half][head][D/4][128 rows] unnormalised O
  float2* part_ml;  // [slot][half][head][128 rows] (running max of y, running sum)
  unsigned* counters;  // [slot], zero on entry
};

// Work items of the CTAs in launch order, longest first: item i covers the
// blocks i*per_tile .. i*per_tile + per_tile - 1 (one per head pair) and
// encodes the query block in bits 2.. and the part in bits 0-1 (0 the whole
// key range, 1 the first half of the key tiles, 2 the second half).
constexpr int kAttnWorkCap = 1920;
struct AttnWork {
  uint16_t item[kAttnWorkCap];
};

// 2^x by the hardware approximation (ex2.approx.ftz.f32, the MUFU unit).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x on the FMA pipe for x <= 8 (Cody-Waite split x = n + f with n = floor(x)
// and f in [0, 1); 2^f by the cubic minimax polynomial 1 + c1 f + c2 f^2 + c3 f^3
// fitted for relative error on [0, 1) (max 8.6e-5); 2^n by adding n to the
// exponent field).  Inputs below -127 return 0.
__device__ __forceinline__ float exp2_poly(float x) {
  x = fmaxf(x, -127.0f);
  const float n = floorf(x);
  const float f = x - n;
  float q = fmaf(f, 0.07706519961357117f, 0.22764700651168823f);
  q = fmaf(q, f, 0.6951163411140442f);
  q = fmaf(q, f, 1.0f);
  return __int_as_float(__float_as_int(q) + (static_cast<int>(n) << 23));
}

// Packed fp32 pairs (two lanes of one 64-bit register): Blackwell executes
// fma/add.f32x2 as one instruction with per-lane IEEE round-to-nearest, so the
// results equal two scalar fmaf/adds.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Two barrier checks issued back to back, so that their shared-memory round
// trips overlap; falls back to the bounded waits when either is still open.
__device__ __forceinline__ bool mbar_wait2(uint64_t* b0, uint32_t p0, uint64_t* b1, uint32_t p1, uint32_t site) {
  const bool r0 = mbar_try_wait(smem_u32(b0), p0);
  const bool r1 = mbar_try_wait(smem_u32(b1), p1);
  if (r0 && r1) return true;
  return mbar_wait(b0, p0, site) && mbar_wait(b1, p1, site);
}

// Epilogue of one softmax warpgroup (128 rows of one query head, O in tensor
// memory at column colO, complete once o_final has been observed): normalise
// and store the output tile through shared memory and TMA; for half of a split
// row block, publish or merge the partial results first (see below).  Shared
// by the attention kernels; `slot` is the split block's slot in p.part.
template <int D>
__device__ __forceinline__ void attn_epilogue(const AttnTcParams& p, const CUtensorMap* tmO, uint8_t* stage_base,
                                              uint32_t tmem, uint32_t lane_base, uint32_t colO, int wg, int row,
                                              int grow, int h, int t, int part_code, int slot, bool ok, float m_run,
                                              float l_run, float gg, volatile uint32_t* abort_flag, int* s_last,
                                              int* s_ready) {
  constexpr int kDBoxes = D / 64;
  const int sw = row & 7;  // 16-byte chunk c of a 128-byte swizzled row sits at c ^ (row & 7)
  float mm = m_run, inv = 0.0f, s_me = 1.0f, s_ot = 0.0f;
  const float4* other = nullptr;
  bool own_first = true;  // merge as fma(O_second, s_second, O_first * s_first) whichever half merges
  bool write_out = ok;
  if (part_code != 0) {
    // half of a split row block.  The slot's counter decides the roles: the
    // half that gets there first (even count) publishes its unnormalised O
    // and (max, sum), then adds 4 (ready); the second (odd count) waits for
    // the ready value 6 = 1 + 1 + 4, merges both and writes the output, so
    // only one fp32 partial makes the round trip through L2.
    const int half = part_code - 1;
    asm volatile("bar.sync 1, 256;" ::: "memory");
    if (threadIdx.x == 0) *s_last = (atomicAdd(&p.counters[slot], 1u) & 1u) ? 1 : 0;
    asm volatile("bar.sync 1, 256;" ::: "memory");
    if (!*s_last) {
      if (ok) {
        float4* mine = p.part + ((static_cast<size_t>(slot) * 2 + half) * 2 + wg) * (D / 4) * 128;
        tc_fence_after();
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_base + colO + c0, o);
          tmem_ld_wait();
#pragma unroll
          for (int v = 0; v < 8; ++v)
            mine[(c0 / 4 + v) * 128 + row] = make_float4(__uint_as_float(o[4 * v]), __uint_as_float(o[4 * v + 1]),
                                                         __uint_as_float(o[4 * v + 2]), __uint_as_float(o[4 * v + 3]));
        }
        p.part_ml[((static_cast<size_t>(slot) * 2 + half) * 2 + wg) * 128 + row] = make_float2(m_run, l_run);
      }
      __threadfence();
      asm volatile("bar.sync 1, 256;" ::: "memory");
      if (threadIdx.x == 0 && !*abort_flag) atomicAdd(&p.counters[slot], 4u);
      write_out = false;
    } else {
      if (threadIdx.x == 0) {
        // bounded wait for the first half's ready value (it is resident and
        // past its own count, so it gets there without this CTA's help)
        bool ready = false;
        const uint64_t t0 = globaltimer_ns();
        for (uint32_t i = 0;; ++i) {
          if (ld_acquire_gpu(&p.counters[slot]) >= 6u) {
            ready = true;
            break;
          }
          if ((i & 63u) == 63u && globaltimer_ns() - t0 > kWaitLimitNs) break;
        }
        if (!ready) {
          raise_error(kErrWaitAttention, 2);
          *abort_flag = 1;
        }
        *s_ready = ready ? 1 : 0;
      }
      asm volatile("bar.sync 1, 256;" ::: "memory");
      write_out = ok && *s_ready;
      if (write_out) {
        __threadfence();
        const size_t ob = (static_cast<size_t>(slot) * 2 + (1 - half)) * 2 + wg;
        const float2 oml = __ldcg(&p.part_ml[ob * 128 + row]);
        other = p.part + ob * (D / 4) * 128;
        own_first = half == 0;
        mm = fmaxf(m_run, oml.x);
        s_me = ex2_approx(gg * (m_run - mm));
        s_ot = ex2_approx(gg * (oml.x - mm));
        // the same rounding whichever half merges: fma(l_second, s_second, l_first * s_first)
        inv = 1.0f / (own_first ? fmaf(oml.y, s_ot, l_run * s_me) : fmaf(l_run, s_me, oml.y * s_ot));
        s_me *= inv;
        s_ot *= inv;
        if (threadIdx.x == 0) p.counters[slot] = 0u;  // ready for the next launch
      }
    }
  } else if (ok) {
    inv = 1.0f / l_run;
    s_me = inv;
  }
  if (write_out) {
    // O as bf16 into the K/V stages, in the
    // 128-byte-swizzled layout of the output tensor map: box b holds columns
    // 64b..64b+63, row r at 128 r, 16-byte chunk c at c ^ (r & 7)
    uint8_t* stage = stage_base + wg * (128 * D * 2);  // idle once o_final has completed
    tc_fence_after();
    // the partner's partial is read one 32-column chunk ahead of its use
    float4 wcur[8];
    if (other) {
#pragma unroll
      for (int v = 0; v < 8; ++v) wcur[v] = __ldcg(&other[v * 128 + row]);
    }
#pragma unroll 1
    for (int c0 = 0; c0 < D; c0 += 32) {
      float4 wnext[8];
      if (other && c0 + 32 < D) {
#pragma unroll
        for (int v = 0; v < 8; ++v) wnext[v] = __ldcg(&other[((c0 + 32) / 4 + v) * 128 + row]);
      }
      uint32_t o[32];
      tmem_ld32(tmem + lane_base + colO + c0, o);
      tmem_ld_wait();
      float f[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) f[e] = __uint_as_float(o[e]) * s_me;
      if (other) {
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          const float4 w4 = wcur[v];
          const float w[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float own = __uint_as_float(o[4 * v + u]);
            f[4 * v + u] = own_first ? fmaf(w[u], s_ot, own * s_me) : fmaf(own, s_me, w[u] * s_ot);
          }
        }
#pragma unroll
        for (int v = 0; v < 8; ++v) wcur[v] = wnext[v];
      }
      uint8_t* box = stage + (c0 / 64) * (128 * 128) + row * 128;
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const int chunk = (c0 % 64) / 8 + v;
        *reinterpret_cast<uint4*>(box + ((chunk ^ sw) << 4)) =
            make_uint4(pack_bf16x2(f[8 * v], f[8 * v + 1]), pack_bf16x2(f[8 * v + 2], f[8 * v + 3]),
                       pack_bf16x2(f[8 * v + 4], f[8 * v + 5]), pack_bf16x2(f[8 * v + 6], f[8 * v + 7]));
      }
    }
    // the warpgroup's tile is staged: one thread stores it (rows past m are clipped)
    fence_proxy_async_smem();
    if (wg == 0) asm volatile("bar.sync 2, 128;" ::: "memory");
    else asm volatile("bar.sync 3, 128;" ::: "memory");
    if (row == 0) {
      for (int b = 0; b < kDBoxes; ++b) tma_store_2d(tmO, stage + b * (128 * 128), h * D + 64 * b, t * 128);
      bulk_commit();
      bulk_wait_all();  // written out before the CTA (and its shared memory) goes away
    }
    if (p.lse && grow < p.m) p.lse[static_cast<int64_t>(h) * p.m + grow] = (gg * mm - log2f(inv)) * kLn2;
  }
}

template <int D>
__global__ void __launch_bounds__(kAttnThreads, 1)
    k_attn_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmBias,
              const __grid_constant__ CUtensorMap tmO, AttnTcParams p, const __grid_constant__ AttnWork work) {
  using Cfg = AttnCfg<D>;
  constexpr int BN = Cfg::BN;
  constexpr int kDBoxes = D / 64;
  extern __shared__ uint8_t attn_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(attn_smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                     // [2 heads][kQBytes]
  uint8_t* sK = smem + Cfg::kOffK;        // [3 stages][kKVBytes]
  uint8_t* sV = smem + Cfg::kOffV;        // [2 stages][kKVBytes]
  float* sBias = reinterpret_cast<float*>(smem + Cfg::kOffBias);  // [3 stages][BN]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kOffBars);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;      // [3]  K tile j (stage j % 3) and its bias tile
  uint64_t* v_full = bars + 4;      // [2]  V tile j (stage j % 2)
  uint64_t* pv_done = bars + 6;     // [4]  P V of tile j (both heads) complete, slot j % 4
  uint64_t* s_full = bars + 10;     // [head * 2 + buffer]
  uint64_t* p_full = bars + 14;     // [head * 2 + buffer]  (128 arrivals: the warpgroup)
  uint64_t* o_final = bars + 18;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 19);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  __shared__ int s_last;
  __shared__ int s_ready;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // longest work first (the last row block has the most causal work)
  const int pairs_per_kv = p.group / 2;
  const int per_tile = p.hkv * pairs_per_kv;
  int t, part_code = 0;
  if (p.use_table) {
    const int it = work.item[blockIdx.x / per_tile];
    t = it >> 2;
    part_code = it & 3;
  } else {
    t = p.num_qtiles - 1 - static_cast<int>(blockIdx.x) / per_tile;
  }
  const int pair = static_cast<int>(blockIdx.x) % per_tile;
  const int g = pair / pairs_per_kv;
  const int h0 = g * p.group + 2 * (pair % pairs_per_kv);
  // causal: key tiles 0 .. (128t + 127) / 64, and none past the last kept row;
  // a split block takes the first or the second half of them
  const int nt_all = min(2 * t + 2, (p.m + BN - 1) / BN);
  const int j0 = part_code == 2 ? nt_all / 2 : 0;
  const int j1 = part_code == 1 ? nt_all / 2 : nt_all;
  const int nt = j1 - j0;  // key tiles of this CTA; local tile i is global tile j0 + i

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < Cfg::kKStages; ++s) mbar_init(&k_full[s], 1);
    for (int s = 0; s < 2; ++s) mbar_init(&v_full[s], 1);
    for (int s = 0; s < 4; ++s) mbar_init(&pv_done[s], 1);
    for (int i = 0; i < 4; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 128);
    }
    mbar_init(o_final, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (!p.has_bias)
    for (int i = threadIdx.x; i < Cfg::kKStages * BN; i += kAttnThreads) sBias[i] = 0.0f;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();
  pdl_launch_dependents();

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      if (p.has_bias) prefetch_tmap(&tmBias);
      mbar_arrive_expect_tx(q_full, 2 * Cfg::kQBytes);
      for (int i = 0; i < 2; ++i)
        for (int b = 0; b < kDBoxes; ++b)
          tma_load_2d(sQ + i * Cfg::kQBytes + b * Cfg::kQBlk, &tmQ, q_full, (h0 + i) * D + 64 * b, t * 128);
      for (int j = 0; j < nt; ++j) {
        // K stage j % 3 held tile j - 3, V stage j % 2 held tile j - 2: both
        // are free once the P V of that tile has completed
        if (j >= 3 && !mbar_wait(&pv_done[(j - 3) & 3], ((j - 3) >> 2) & 1, kErrWaitAttention)) {
          *abort_flag = 1;
          break;
        }
        const int ks = j % 3, vs = j & 1;
        mbar_arrive_expect_tx(&k_full[ks], Cfg::kKVBytes + (p.has_bias ? BN * 4 : 0));
        for (int b = 0; b < kDBoxes; ++b)
          tma_load_2d(sK + ks * Cfg::kKVBytes + b * Cfg::kKVBlk, &tmK, &k_full[ks], g * D + 64 * b, (j0 + j) * BN);
        if (p.has_bias) tma_load_1d(sBias + ks * BN, &tmBias, &k_full[ks], (j0 + j) * BN);
        if (j >= 2 && !mbar_wait(&pv_done[(j - 2) & 3], ((j - 2) >> 2) & 1, kErrWaitAttention)) {
          *abort_flag = 1;
          break;
        }
        mbar_arrive_expect_tx(&v_full[vs], Cfg::kKVBytes);
        for (int b = 0; b < kDBoxes; ++b)
          tma_load_2d(sV + vs * Cfg::kKVBytes + b * Cfg::kKVBlk, &tmV, &v_full[vs], g * D + 64 * b, (j0 + j) * BN);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, BN, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, false, true);
      // descriptors of every operand's first 16-element K slice; a later
      // slice adds its byte offset / 16 to the start-address field
      const uint64_t dq0 = sdesc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dk0 = sdesc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t dv0 = sdesc_sw128(smem_u32(sV), Cfg::kKVBlk, 1024);
      auto issue_qk = [&](int h, int j) {
        const uint64_t da = dq0 + (h * Cfg::kQBytes >> 4), db = dk0 + ((j % 3) * Cfg::kKVBytes >> 4);
        const uint32_t d_tmem = tmem + attn_col_s(h, j & 1);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_ss(d_tmem, da + (((kk >> 2) * Cfg::kQBlk + (kk & 3) * 32) >> 4),
                  db + (((kk >> 2) * Cfg::kKVBlk + (kk & 3) * 32) >> 4), idesc_qk, kk != 0 ? 1u : 0u);
        umma_commit(&s_full[2 * h + (j & 1)]);
      };
      auto issue_pv = [&](int h, int j) {
        // A = P from tensor memory (two bf16 keys per column, over the S columns of tile j)
        const uint32_t pa = tmem + attn_col_s(h, j & 1);
        const uint64_t db = dv0 + ((j & 1) * Cfg::kKVBytes >> 4);
        const uint32_t d_tmem = tmem + (h ? Cfg::kColO1 : Cfg::kColO0);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          umma_ts(d_tmem, pa + kk * 8, db + ((kk * 16 * 128) >> 4), idesc_pv, (j | kk) != 0 ? 1u : 0u);
      };
      // the scores of tiles 0 and 1 first
      bool ok = mbar_wait2(q_full, 0, &k_full[0], 0, kErrWaitAttention);
      if (ok) {
        tc_fence_after();
        issue_qk(0, 0);
        issue_qk(1, 0);
      }
      if (ok && nt > 1 && (ok = mbar_wait(&k_full[1], 0, kErrWaitAttention))) {
        tc_fence_after();
        issue_qk(0, 1);
        issue_qk(1, 1);
      }
      // per tile j: P V of tile j for head 0, then head 1, then the scores of
      // tile j + 2 into the S buffers whose tile j the softmax has read (its
      // p_full arrival comes after its S loads completed)
      // Each barrier check of this thread holds back its next MMA issue for a
      // shared-memory round trip (~150-250 cycles), during which the tensor
      // core's short queue drains; so all four barriers a tile needs (V, the P
      // of both heads, K of tile j + 2) are checked at once, and the tile's
      // twenty-four MMAs then issue back to back.
      for (int j = 0; ok && j < nt; ++j) {
        const uint32_t ph = (j >> 1) & 1;
        const bool next = j + 2 < nt;
        {
          uint64_t* kb = &k_full[(j + 2) % 3];
          const uint32_t kph = ((j + 2) / 3) & 1;
          const bool r0 = mbar_try_wait(smem_u32(&v_full[j & 1]), ph);
          const bool r1 = mbar_try_wait(smem_u32(&p_full[j & 1]), ph);
          const bool r2 = mbar_try_wait(smem_u32(&p_full[2 + (j & 1)]), ph);
          const bool r3 = !next || mbar_try_wait(smem_u32(kb), kph);
          if (!(r0 && r1 && r2 && r3)) {
            ok = mbar_wait2(&v_full[j & 1], ph, &p_full[j & 1], ph, kErrWaitAttention) &&
                 mbar_wait(&p_full[2 + (j & 1)], ph, kErrWaitAttention) &&
                 (!next || mbar_wait(kb, kph, kErrWaitAttention));
            if (!ok) break;
          }
        }
        tc_fence_after();
        issue_pv(0, j);
        issue_pv(1, j);
        umma_commit(&pv_done[j & 3]);
        if (next) {
          issue_qk(0, j + 2);
          issue_qk(1, j + 2);
        }
      }
      if (ok) umma_commit(o_final);
      else *abort_flag = 1;
    }
  } else {
    // ------------------------------------------------------------ softmax warpgroups
    const int wg = warp >> 2;           // 0 or 1: which query head
    const int q4 = warp & 3;            // TMEM lane quarter
    const int row = q4 * 32 + lane;     // row inside the query tile
    const int grow = t * 128 + row;
    const int h = h0 + wg;
    const uint32_t colO = wg ? Cfg::kColO1 : Cfg::kColO0;
    const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
    const float a_row = grow < p.m ? p.temp[h] * (p.ratio ? p.ratio[grow] : 1.0f) * p.scale_log2 : 0.0f;
    // g > 0 always (a zero gain leaves the bias term at 1e-20 * bias, i.e. nothing)
    const float gg = fmaxf(p.gain[h] * kLog2e, 1e-20f);
    const float a_y = a_row / gg;
    const uint64_t ay2 = f2_pack(a_y, a_y), gg2 = f2_pack(gg, gg);
    float m_run = -INFINITY, l_run = 0.0f;  // running max of y, running sum of exp2(g * (y - m_run))
    bool ok = true;

    for (int j = 0; j < nt; ++j) {
      const int b = j & 1;
      const uint32_t ph = (j >> 1) & 1;
      // S of tile j and its bias tile (it rides with K); P goes over the S
      // columns, which the P V of tile j - 2 had read before the Q K^T of
      // tile j wrote them
      bool rdy = !*abort_flag && mbar_wait2(&s_full[2 * wg + b], ph, &k_full[j % 3], (j / 3) & 1, kErrWaitAttention);
      if (!__all_sync(0xffffffffu, rdy)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t s0[32], s1[32];
      tmem_ld32(tmem + lane_base + attn_col_s(wg, b), s0);
      tmem_ld32(tmem + lane_base + attn_col_s(wg, b) + 32, s1);
      tmem_ld_wait();
      const float* bias = sBias + (j % 3) * BN;
      // Pass 1: y = a_y * S + bias on pairs, and the row maximum (four
      // independent chains); the causal mask only touches the key tiles that
      // cross the diagonal.
      uint64_t y2[BN / 2];
      const int key0 = (j0 + j) * BN;
      const bool diag = key0 + BN - 1 > t * 128;  // warp-uniform
      float mxv[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      auto logits = [&](const uint32_t(&r)[32], int c0) {
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const float4 b4 = *reinterpret_cast<const float4*>(bias + c0 + e);
          const int i = (c0 + e) >> 1;
          y2[i] = f2_fma(ay2, f2_pack(__uint_as_float(r[e]), __uint_as_float(r[e + 1])), f2_pack(b4.x, b4.y));
          y2[i + 1] = f2_fma(ay2, f2_pack(__uint_as_float(r[e + 2]), __uint_as_float(r[e + 3])), f2_pack(b4.z, b4.w));
          if (diag) {
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              float lo, hi;
              f2_unpack(y2[i + u], lo, hi);
              const int c = key0 + c0 + e + 2 * u;
              if (c > grow) lo = -INFINITY;
              if (c + 1 > grow) hi = -INFINITY;
              y2[i + u] = f2_pack(lo, hi);
            }
          }
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            float lo, hi;
            f2_unpack(y2[i + u], lo, hi);
            mxv[(i + u) & 3] = fmax3(mxv[(i + u) & 3], lo, hi);
          }
        }
      };
      logits(s0, 0);
      logits(s1, 32);
      const float mx = fmaxf(fmaxf(mxv[0], mxv[1]), fmaxf(mxv[2], mxv[3]));
      // lazy rescaling: the reference maximum only moves when the row maximum
      // exceeds it by more than 8 in log2 units, so every p stays <= 2^8
      // (per row: the branch is divergent, so it holds no warp-collective op)
      float sc = 1.0f;
      if (gg * (mx - m_run) > 8.0f) {
        if (j > 0) sc = ex2_approx(gg * (m_run - mx));
        m_run = mx;
      }
      const float nm = -gg * m_run;
      const uint64_t nm2 = f2_pack(nm, nm);
      // Pass 2: p = 2^(g*y - g*m), partial sums on pairs, P as bf16 pairs into
      // tensor memory over the first 32 columns of this tile's S buffer
      uint64_t sum2[2] = {0, 0};
      uint32_t pk[BN / 2];
#pragma unroll
      for (int i = 0; i < BN / 2; ++i) {
        float x0, x1;
        f2_unpack(f2_fma(gg2, y2[i], nm2), x0, x1);
        float p0, p1;
        if (kPolyShare && (i & 3) == 3) {
          p0 = exp2_poly(x0);
          p1 = exp2_poly(x1);
        } else {
          p0 = ex2_approx(x0);
          p1 = ex2_approx(x1);
        }
        sum2[i & 1] = f2_add(sum2[i & 1], f2_pack(p0, p1));
        pk[i] = pack_bf16x2(p0, p1);
      }
      tmem_st32(tmem + lane_base + attn_col_s(wg, b), pk);
      float sa, sb, sc2, sd;
      f2_unpack(sum2[0], sa, sb);
      f2_unpack(sum2[1], sc2, sd);
      l_run = l_run * sc + ((sa + sb) + (sc2 + sd));
      // tcgen05.ld/st are warp-collective (.sync.aligned): the whole warp
      // rescales its 32 rows if any of them needs it, the others with sc = 1
      if (__any_sync(0xffffffffu, sc != 1.0f)) {
        // O holds the sum over tiles < j once the P V of tile j - 1 is done;
        // the P V of tile j is not issued before p_full below
        if (!warp_wait(&pv_done[(j - 1) & 3], ((j - 1) >> 2) & 1, kErrWaitAttention)) {
          ok = false;
          break;
        }
        tc_fence_after();
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
      // the S loads, the P store and any O rescale are complete: hand P over
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_full[2 * wg + b]);
    }
    if (ok && !*abort_flag) ok = warp_wait(o_final, 0, kErrWaitAttention);
    // every softmax thread ends here, so the named barriers below see all 256
    if (!ok) *abort_flag = 1;
    attn_epilogue<D>(p, &tmO, sK, tmem, lane_base, colO, wg, row, grow, h, t, part_code, (t - p.ts) * per_tile + pair, ok,
                     m_run, l_run, gg, abort_flag, &s_last, &s_ready);
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

// Token-gated causal GQA flash attention on the 5th-generation tensor cores.
//
// Method ("TokenGate and T2Quant: a close reading", §4.1 token-gated
// attention, head-wise gain, temperature scaling): for query head h, KV head g
// and kept rows c <= r
//     l_rc = temp_h * ratio_r * sm_scale * (q_r . k_c) + gain_h * bias_c
//     o_r  = sum_c softmax_c(l_r.) v_c
// computed in base 2, x_rc = l_rc * log2(e) = a_r * S'_rc, with
//     a_r = temp_h * ratio_r * sm_scale * log2(e),   g_h = gain_h * log2(e),
//     S'_rc = q_r . k_c + u_r * bias_c,   u_r = g_h / a_r.
// The key bias enters the score MMA itself: each Q K^T gets one more K = 16
// MMA of E_h F^T, where row r of E_h is (u_hi, u_hi, u_lo, 0 ...) and key row c
// of F is (b_hi, b_lo, b_hi, 0 ...) (bf16 hi/lo splits of u_r and bias_c, so
// u_r * bias_c is carried to about 2^-17 relative), so the softmax reads
// nothing from shared memory, whose bandwidth the score MMAs need.  |a_r| is
// held at least 1e-30 (a zero content scale then leaves 1e-30 * S, nothing).
//
// One CTA owns a 128-row query block of TWO query heads that share a KV head
// (GQA), so every K/V tile fetched by TMA feeds two score tiles.  Keys come in
// tiles of 128, so each Q K^T is an M128 N128 MMA (an N64 one is bound by the
// shared-memory reads of its A operand).
//   warps 0-3  softmax warpgroup 0 (query head 0), one thread per row; at
//              the start each thread writes its row of E_0
//   warps 4-7  softmax warpgroup 1 (query head 1), and E_1
//   warp 8     TMA producer (Q once; K and V tiles through two-stage rings,
//              the fp32 bias through a four-stage staging ring) and, all 32
//              lanes, the conversion of each bias tile into F
//   warp 9     TMEM allocator and single-thread tcgen05.mma issuer
// Tensor memory (512 columns): S0 | S1 (128 columns each), O0 | O1 (D each).
// S' is an SS-MMA into TMEM; the softmax reads it with tcgen05.ld and writes
// P = exp2(x - m) as bf16 pairs over the first 64 columns of the same S
// buffer; O += P V is a TS-MMA (P from tensor memory, V MN-major from shared
// memory).
//
// The two heads take turns (ping-pong): per key tile j the MMA thread issues
//     P0 V(j), Q0 K(j+1)^T, P1 V(j), Q1 K(j+1)^T
// so while one warpgroup turns its scores into probabilities the tensor core
// works on the other head, and the loop is bound by the slower of the tensor
// core (four M128 N128 K128 products per tile) and one head's softmax, not by
// their sum.  Because the scores of head i for tile j+1 are issued after its
// P V of tile j, their completion (the s_full barrier) also means that P V is
// done: the softmax rescales O in place when its running maximum moves
// without waiting for anything.  The running maximum only moves when it grows
// by more than 8 (log2 units), so every p stays <= 2^8.
//
// Exponentials: two heads of 128 x 128 probabilities per tile are as many
// MUFU operations (16 per clock per SM) as the tensor core has cycles, so one
// pair in four off the diagonal is evaluated on the FMA pipe instead
// (exp2_poly2), leaving the MUFU unit headroom.  The elementwise arithmetic
// runs on packed pairs (fma/add.f32x2, three-input max).
#pragma once

#include <type_traits>

#include "common.cuh"
#include "simt.cuh"

namespace tg {

constexpr int kAttnThreads = 320;

template <int D>
struct AttnCfg {
  static constexpr int BM = 128, BN = 128;
  static constexpr int kQBytes = BM * D * 2;     // one query tile
  static constexpr int kKVBytes = BN * D * 2;    // one K or V tile
  static constexpr int kQBlk = BM * 128;         // one 64-column TMA box of a Q tile
  static constexpr int kKVBlk = BN * 128;        // one 64-column TMA box of a K or V tile
  static constexpr int kStages = 2;              // K ring and V ring (and F)
  static constexpr int kBiasStages = 4;          // fp32 bias staging ring
  static constexpr int kExtBytes = 128 * 32;     // E_h or one F tile: 128 rows x 16 bf16
  static constexpr int kColO0 = 2 * BN, kColO1 = 2 * BN + D;
  static constexpr size_t kOffK = 2 * kQBytes;
  static constexpr size_t kOffV = kOffK + kStages * kKVBytes;
  static constexpr size_t kOffE = kOffV + kStages * kKVBytes;      // [2 heads][kExtBytes]
  static constexpr size_t kOffF = kOffE + 2 * kExtBytes;           // [2 stages][kExtBytes]
  static constexpr size_t kOffBias = kOffF + kStages * kExtBytes;  // [4 stages][BN] fp32
  static constexpr size_t kOffBars = kOffBias + kBiasStages * BN * 4;  // 19 barriers + TMEM slot
  static constexpr size_t kData = kOffBars + 256;
  // D = 64 is padded so that only one CTA fits on an SM and its 512-column
  // TMEM allocation never waits on a neighbour
  static constexpr size_t kSmem = 1024 + (kData < 120 * 1024 ? 120 * 1024 : kData);
};

// TMEM column of head h's S buffer (and of its P, over the first BN/2 columns)
__device__ __forceinline__ uint32_t attn_col_s(int h) { return static_cast<uint32_t>(h * 128); }

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

// Coefficients of q(u) ~ 2^(u + 1/2) on [-1/2, 1/2]: the cubic minimax
// polynomial for relative error (Remez exchange; max 7.5e-5).
constexpr float kExp2C0 = 1.414111852645874f;
constexpr float kExp2C1 = 0.9804190993309021f;
constexpr float kExp2C2 = 0.34310394525527954f;
constexpr float kExp2C3 = 0.07802452147006989f;

// 2^x of a pair on the FMA pipe, given xh = x - 1/2 with x <= 8 (lanes below
// -125 are clamped there, so every result is a normal float).  Cody-Waite
// split xh = n + u with n the nearest
// integer (adding and subtracting 1.5 * 2^23 rounds it into the low mantissa
// bits) and u in [-1/2, 1/2]; 2^(u + 1/2) = q(u); 2^n by adding n to the
// exponent field of q, which is the low bits of the rounded sum shifted up
// by 23.
__device__ __forceinline__ uint64_t exp2_poly2(uint64_t xh2) {
  float a, b;
  f2_unpack(xh2, a, b);
  const uint64_t x2 = f2_pack(fmaxf(a, -125.5f), fmaxf(b, -125.5f));
  const uint64_t t2 = f2_add(x2, f2_pack(12582912.0f, 12582912.0f));
  const uint64_t n2 = f2_add(t2, f2_pack(-12582912.0f, -12582912.0f));
  const uint64_t u2 = f2_fma(n2, f2_pack(-1.0f, -1.0f), x2);
  uint64_t q2 = f2_fma(f2_pack(kExp2C3, kExp2C3), u2, f2_pack(kExp2C2, kExp2C2));
  q2 = f2_fma(q2, u2, f2_pack(kExp2C1, kExp2C1));
  q2 = f2_fma(q2, u2, f2_pack(kExp2C0, kExp2C0));
  float q0, q1, t0, t1;
  f2_unpack(q2, q0, q1);
  f2_unpack(t2, t0, t1);
  return f2_pack(__int_as_float(__float_as_int(q0) + (__float_as_int(t0) << 23)),
                 __int_as_float(__float_as_int(q1) + (__float_as_int(t1) << 23)));
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
        const uint32_t target = g_merge_ready_target;
        const uint64_t limit = g_flag_wait_limit_ns;
        const uint64_t t0 = globaltimer_ns();
        for (uint32_t i = 0;; ++i) {
          if (ld_acquire_gpu(&p.counters[slot]) >= target) {
            ready = true;
            break;
          }
          if ((i & 63u) == 63u && globaltimer_ns() - t0 > limit) break;
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

// One softmax warpgroup thread's share of a key tile: its query row against
// the tile's 128 keys, x = a * S' read from tensor memory twice in groups of
// 32 columns, the next group's load issued before the current group is
// processed (its wait comes after, so the latency hides behind arithmetic):
//   pass 1: the row maximum of x (four chains);
//   lazy rescale: the reference maximum only moves when the row maximum
//     exceeds it by more than 8, so every p stays <= 2^8; when any row of the
//     warp moves, the warp rescales its rows of O in tensor memory (the P V
//     that last wrote O is complete, see the kernel);
//   pass 2: p = 2^(x - m), the row sum (four chains) and P as bf16 pairs over
//     S columns already read (the P of keys 32q .. 32q + 31 goes to columns
//     16q .. 16q + 15).
// kDiag: the tile crosses the diagonal, keys past the row are masked with
// -inf and every exponential goes to the MUFU unit (exp2(-inf) = 0 exactly);
// off the diagonal one pair in four is evaluated on the FMA pipe.
// The tile's second pass: P = exp2(a S' - m) for the row's maximum m (nm2 =
// -m, nmh2 = -m - 1/2 for the FMA-pipe form) written back as bf16 pairs over
// the first 64 columns of the same S buffer; returns the row sum of P.
template <bool kDiag>
__device__ __forceinline__ float attn_exp_pass(uint32_t t_s, uint64_t a2, uint64_t nm2, uint64_t nmh2, int key0,
                                               int grow) {
  constexpr int BN = 128, G = BN / 32;
  uint64_t sum2[4] = {0, 0, 0, 0};
  uint32_t buf[2][32];
  tmem_ld32(t_s, buf[0]);
  tmem_ld_wait();
#pragma unroll
  for (int q = 0; q < G; ++q) {
    if (q + 1 < G) tmem_ld32(t_s + 32 * (q + 1), buf[(q + 1) & 1]);
    const uint32_t* r = buf[q & 1];
    uint32_t pk[16];
#pragma unroll
    for (int v = 0; v < 16; ++v) {
      const int e = 2 * v;  // keys 32q + e and 32q + e + 1
      float s0 = __uint_as_float(r[e]), s1 = __uint_as_float(r[e + 1]);
      if (kDiag) {
        const int k = key0 + 32 * q + e;
        if (k > grow) s0 = -INFINITY;
        if (k + 1 > grow) s1 = -INFINITY;
      }
      const uint64_t s2 = f2_pack(s0, s1);
      uint64_t p2;
      if (!kDiag && (v & 3) == 3) {
        p2 = exp2_poly2(f2_fma(a2, s2, nmh2));
      } else {
        float x0, x1;
        f2_unpack(f2_fma(a2, s2, nm2), x0, x1);
        p2 = f2_pack(ex2_approx(x0), ex2_approx(x1));
      }
      sum2[v & 3] = f2_add(sum2[v & 3], p2);
      float p0, p1;
      f2_unpack(p2, p0, p1);
      pk[v] = pack_bf16x2(p0, p1);
    }
    tmem_st16(t_s + 16 * q, pk);
    if (q + 1 < G) tmem_ld_wait();
  }
  float a0, a1, b0, b1;
  f2_unpack(f2_add(sum2[0], sum2[1]), a0, a1);
  f2_unpack(f2_add(sum2[2], sum2[3]), b0, b1);
  return (a0 + a1) + (b0 + b1);
}

template <int D, bool kDiag>
__device__ __forceinline__ void attn_softmax_tile(uint32_t t_s, uint32_t t_o, uint64_t a2, int key0, int grow,
                                                  bool first, float& m_run, float& l_run) {
  constexpr int BN = 128, G = BN / 32;
  float a, a_hi;
  f2_unpack(a2, a, a_hi);
  // The tile's maximum of x = a S': for a > 0 it is a * max(S') exactly (the
  // rounding of a product is monotonic in the other factor), which saves the
  // scaling of every element in this pass; otherwise the scaled values.
  float mx;
  {
    const bool raw = __all_sync(0xffffffffu, a > 0.0f);
    const uint64_t zero2 = f2_pack(0.0f, 0.0f);
    float mxv[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
    uint32_t buf[2][32];
    tmem_ld32(t_s, buf[0]);
    tmem_ld_wait();
#pragma unroll
    for (int q = 0; q < G; ++q) {
      if (q + 1 < G) tmem_ld32(t_s + 32 * (q + 1), buf[(q + 1) & 1]);
      const uint32_t* r = buf[q & 1];
#pragma unroll
      for (int e = 0; e < 32; e += 4) {
        float l0 = __uint_as_float(r[e]), h0 = __uint_as_float(r[e + 1]);
        float l1 = __uint_as_float(r[e + 2]), h1 = __uint_as_float(r[e + 3]);
        if (!raw) {
          f2_unpack(f2_fma(a2, f2_pack(l0, h0), zero2), l0, h0);
          f2_unpack(f2_fma(a2, f2_pack(l1, h1), zero2), l1, h1);
        }
        if (kDiag) {
          const int k = key0 + 32 * q + e;
          if (k > grow) l0 = -INFINITY;
          if (k + 1 > grow) h0 = -INFINITY;
          if (k + 2 > grow) l1 = -INFINITY;
          if (k + 3 > grow) h1 = -INFINITY;
        }
        mxv[(e >> 2) & 3] = fmax3(mxv[(e >> 2) & 3], fmaxf(l0, h0), fmaxf(l1, h1));
      }
      if (q + 1 < G) tmem_ld_wait();
    }
    mx = fmaxf(fmaxf(mxv[0], mxv[1]), fmaxf(mxv[2], mxv[3]));
    if (raw) mx = a * mx;
  }
  float sc = 1.0f;
  if (mx - m_run > 8.0f) {  // per row: divergent, so no warp-collective op inside
    if (!first) sc = ex2_approx(m_run - mx);
    m_run = mx;
  }
  // tcgen05.ld/st are warp-collective (.sync.aligned): the whole warp rescales
  // its 32 rows if any of them needs it, the others with sc = 1
  if (__any_sync(0xffffffffu, sc != 1.0f)) {
#pragma unroll 1
    for (int c0 = 0; c0 < D; c0 += 32) {
      uint32_t o[32];
      tmem_ld32(t_o + c0, o);
      tmem_ld_wait();
#pragma unroll
      for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * sc);
      tmem_st32(t_o + c0, o);
    }
  }
  const float sum =
      attn_exp_pass<kDiag>(t_s, a2, f2_pack(-m_run, -m_run), f2_pack(-m_run - 0.5f, -m_run - 0.5f), key0, grow);
  l_run = l_run * sc + sum;
}

// bf16 hi/lo split: v ~= hi + lo, both bf16 (rounded to nearest)
__device__ __forceinline__ void bf16_split(float v, __nv_bfloat16& hi, __nv_bfloat16& lo) {
  hi = __float2bfloat16_rn(v);
  lo = __float2bfloat16_rn(v - __bfloat162float(hi));
}

// Row r of a 32-byte-swizzled K = 16 operand tile: (x, y, z, 0 x 13) in bf16
__device__ __forceinline__ void write_ext_row(uint8_t* tile, int r, __nv_bfloat16 x, __nv_bfloat16 y,
                                              __nv_bfloat16 z) {
  __nv_bfloat162 xy, z0;
  xy.x = x;
  xy.y = y;
  z0.x = z;
  z0.y = __float2bfloat16_rn(0.0f);
  *reinterpret_cast<uint4*>(tile + sw32_offset(r, 0)) =
      make_uint4(*reinterpret_cast<uint32_t*>(&xy), *reinterpret_cast<uint32_t*>(&z0), 0u, 0u);
  *reinterpret_cast<uint4*>(tile + sw32_offset(r, 1)) = make_uint4(0u, 0u, 0u, 0u);
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
  uint8_t* sK = smem + Cfg::kOffK;        // [2 stages][kKVBytes]
  uint8_t* sV = smem + Cfg::kOffV;        // [2 stages][kKVBytes]
  uint8_t* sE = smem + Cfg::kOffE;        // [2 heads][kExtBytes]   rows (u_hi, u_hi, u_lo)
  uint8_t* sF = smem + Cfg::kOffF;        // [2 stages][kExtBytes]  key rows (b_hi, b_lo, b_hi)
  float* sBias = reinterpret_cast<float*>(smem + Cfg::kOffBias);  // [4 stages][BN] fp32
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Cfg::kOffBars);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;      // [2]  K tile j and F tile j in stage j % 2 (TMA bytes + the converter)
  uint64_t* k_free = bars + 3;      // [2]  both heads' Q K^T of that tile complete
  uint64_t* v_full = bars + 5;      // [2]  V tile j in stage j % 2
  uint64_t* v_free = bars + 7;      // [2]  both heads' P V of that tile complete
  uint64_t* s_full = bars + 9;      // [head]  S' of the head's current tile (and every earlier MMA) complete
  uint64_t* p_full = bars + 11;     // [head]  P written (128 arrivals: the warpgroup)
  uint64_t* o_final = bars + 13;
  uint64_t* b_full = bars + 14;     // [4]  fp32 bias tile j in staging stage j % 4
  uint64_t* e_full = bars + 18;     // E_0 and E_1 written (256 arrivals)
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
  // causal: key tiles 0 .. t (rows 128t .. 128t + 127), and none past the last
  // kept row; a split block takes the first or the second half of them
  const int nt_all = min(t + 1, (p.m + BN - 1) / BN);
  const int j0 = part_code == 2 ? nt_all / 2 : 0;
  const int j1 = part_code == 1 ? nt_all / 2 : nt_all;
  const int nt = j1 - j0;  // key tiles of this CTA; local tile i is global tile j0 + i

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], 2);
      mbar_init(&k_free[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_free[s], 1);
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], 128);
    }
    for (int s = 0; s < Cfg::kBiasStages; ++s) mbar_init(&b_full[s], 1);
    mbar_init(o_final, 1);
    mbar_init(e_full, 256);
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
  pdl_wait();
  pdl_launch_dependents();

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer + F conversion
    bool ok = true;
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      if (p.has_bias) prefetch_tmap(&tmBias);
      mbar_arrive_expect_tx(q_full, 2 * Cfg::kQBytes);
      for (int i = 0; i < 2; ++i)
        for (int b = 0; b < kDBoxes; ++b)
          tma_load_2d(sQ + i * Cfg::kQBytes + b * Cfg::kQBlk, &tmQ, q_full, (h0 + i) * D + 64 * b, t * 128);
      if (p.has_bias)
        for (int j = 0; j < 2 && j < nt; ++j) {
          mbar_arrive_expect_tx(&b_full[j], BN * 4);
          tma_load_1d(sBias + j * BN, &tmBias, &b_full[j], (j0 + j) * BN);
        }
    }
    for (int j = 0; j < nt; ++j) {
      // stage j % 2 held tile j - 2: K (and F) are free once both heads'
      // Q K^T of that tile completed, V once both P V did
      const int s = j & 1;
      const uint32_t fph = ((j - 2) >> 1) & 1;
      if (lane == 0) {
        if (j >= 2 && !mbar_wait(&k_free[s], fph, kErrWaitAttention)) {
          ok = false;
        } else {
          mbar_arrive_expect_tx(&k_full[s], Cfg::kKVBytes);
          for (int b = 0; b < kDBoxes; ++b)
            tma_load_2d(sK + s * Cfg::kKVBytes + b * Cfg::kKVBlk, &tmK, &k_full[s], g * D + 64 * b, (j0 + j) * BN);
          if (j >= 2 && !mbar_wait(&v_free[s], fph, kErrWaitAttention)) {
            ok = false;
          } else {
            mbar_arrive_expect_tx(&v_full[s], Cfg::kKVBytes);
            for (int b = 0; b < kDBoxes; ++b)
              tma_load_2d(sV + s * Cfg::kKVBytes + b * Cfg::kKVBlk, &tmV, &v_full[s], g * D + 64 * b,
                          (j0 + j) * BN);
          }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      if (p.has_bias) {
        // F(j) from the fp32 bias tile: lane l converts keys 4l .. 4l + 3
        const int bs = j & 3;
        if (!warp_wait(&b_full[bs], (j >> 2) & 1, kErrWaitAttention)) {
          ok = false;
          break;
        }
        const float4 b4 = *reinterpret_cast<const float4*>(sBias + bs * BN + 4 * lane);
        const float bv[4] = {b4.x, b4.y, b4.z, b4.w};
        uint8_t* f = sF + s * Cfg::kExtBytes;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          __nv_bfloat16 hi, lo;
          bf16_split(bv[u], hi, lo);
          write_ext_row(f, 4 * lane + u, hi, lo, hi);
        }
        fence_proxy_async_smem();
        __syncwarp();
        // staging stage (j + 2) % 4 last held tile j - 2, converted two steps ago
        if (lane == 0 && j + 2 < nt) {
          mbar_arrive_expect_tx(&b_full[(j + 2) & 3], BN * 4);
          tma_load_1d(sBias + ((j + 2) & 3) * BN, &tmBias, &b_full[(j + 2) & 3], (j0 + j + 2) * BN);
        }
      }
      if (lane == 0) mbar_arrive(&k_full[s]);  // F(j) written (or no bias to add)
    }
    if (!ok) *abort_flag = 1;
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
      const uint64_t de0 = sdesc_sw32(smem_u32(sE)), df0 = sdesc_sw32(smem_u32(sF));
      const bool ext = p.has_bias != 0;
      auto issue_qk = [&](int h, int j) {
        const uint64_t da = dq0 + (h * Cfg::kQBytes >> 4), db = dk0 + ((j & 1) * Cfg::kKVBytes >> 4);
        const uint32_t d_tmem = tmem + attn_col_s(h);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_ss(d_tmem, da + (((kk >> 2) * Cfg::kQBlk + (kk & 3) * 32) >> 4),
                  db + (((kk >> 2) * Cfg::kKVBlk + (kk & 3) * 32) >> 4), idesc_qk, kk != 0 ? 1u : 0u);
        // + E_h F(j)^T: the key bias times u_r
        if (ext)
          umma_ss(d_tmem, de0 + ((h * Cfg::kExtBytes) >> 4), df0 + (((j & 1) * Cfg::kExtBytes) >> 4), idesc_qk, 1u);
        umma_commit(&s_full[h]);
      };
      auto issue_pv = [&](int h, int j) {
        // A = P from tensor memory (two bf16 keys per column, over the S columns)
        const uint32_t pa = tmem + attn_col_s(h);
        const uint64_t db = dv0 + ((j & 1) * Cfg::kKVBytes >> 4);
        const uint32_t d_tmem = tmem + (h ? Cfg::kColO1 : Cfg::kColO0);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          umma_ts(d_tmem, pa + kk * 8, db + ((kk * 16 * 128) >> 4), idesc_pv, (j | kk) != 0 ? 1u : 0u);
      };
      // the scores of tile 0 for both heads first
      bool ok = mbar_wait2(q_full, 0, &k_full[0], 0, kErrWaitAttention) && mbar_wait(e_full, 0, kErrWaitAttention);
      if (ok) {
        tc_fence_after();
        issue_qk(0, 0);
        issue_qk(1, 0);
        umma_commit(&k_free[0]);
      }
      // per tile j: P0 V(j) and Q0 K(j+1)^T once V(j), P0(j) and K(j+1) are
      // there (checked together: each barrier check holds back the next MMA
      // issue for a shared-memory round trip); then P1 V(j) and Q1 K(j+1)^T
      // once P1(j) is.  Q_i K(j+1)^T overwrites S_i / P_i after P_i V(j) has
      // read P_i (tcgen05 MMAs of one thread run in issue order).
      for (int j = 0; ok && j < nt; ++j) {
        const int s = j & 1;
        const uint32_t vph = (j >> 1) & 1, pph = j & 1;
        const bool next = j + 1 < nt;
        uint64_t* kb = &k_full[(j + 1) & 1];
        const uint32_t kph = ((j + 1) >> 1) & 1;
        {
          const bool r0 = mbar_try_wait(smem_u32(&v_full[s]), vph);
          const bool r1 = mbar_try_wait(smem_u32(&p_full[0]), pph);
          const bool r2 = !next || mbar_try_wait(smem_u32(kb), kph);
          if (!(r0 && r1 && r2)) {
            ok = mbar_wait2(&v_full[s], vph, &p_full[0], pph, kErrWaitAttention) &&
                 (!next || mbar_wait(kb, kph, kErrWaitAttention));
            if (!ok) break;
          }
        }
        tc_fence_after();
        issue_pv(0, j);
        if (next) issue_qk(0, j + 1);
        if (!mbar_try_wait(smem_u32(&p_full[1]), pph) && !(ok = mbar_wait(&p_full[1], pph, kErrWaitAttention)))
          break;
        tc_fence_after();
        issue_pv(1, j);
        umma_commit(&v_free[s]);
        if (next) {
          issue_qk(1, j + 1);
          umma_commit(&k_free[(j + 1) & 1]);
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
    const uint32_t colS = attn_col_s(wg);
    const uint32_t colO = wg ? Cfg::kColO1 : Cfg::kColO0;
    const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
    // x = a * S' with S' = q . k + u * bias, u = g / a (|a| held >= 1e-30)
    float a_row = grow < p.m ? p.temp[h] * (p.ratio ? p.ratio[grow] : 1.0f) * p.scale_log2 : 0.0f;
    if (fabsf(a_row) < 1e-30f) a_row = 1e-30f;
    {
      __nv_bfloat16 uh, ul;
      bf16_split(p.gain[h] * kLog2e / a_row, uh, ul);
      write_ext_row(sE + wg * Cfg::kExtBytes, row, uh, uh, ul);
      fence_proxy_async_smem();
      mbar_arrive(e_full);
    }
    const uint64_t a2 = f2_pack(a_row, a_row);
    float m_run = -INFINITY, l_run = 0.0f;  // running max of x, running sum of exp2(x - m_run)
    bool ok = true;

    // one key tile: wait for its scores (the s_full phase completes once per
    // tile), turn them into P, hand P over once the S loads, the P stores and
    // any O rescale are done
    auto tile = [&](int j, auto diag) -> bool {
      bool rdy = !*abort_flag && mbar_wait(&s_full[wg], j & 1, kErrWaitAttention);
      if (!__all_sync(0xffffffffu, rdy)) return false;
      tc_fence_after();
      attn_softmax_tile<D, decltype(diag)::value>(tmem + lane_base + colS, tmem + lane_base + colO, a2,
                                                  (j0 + j) * BN, grow, j == 0, m_run, l_run);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&p_full[wg]);
      return true;
    };
    // only global tile t crosses the diagonal (keys 128t .. 128t + 127), and
    // when this CTA has it, it is its last tile; the masked variant of the
    // tile is kept out of the loop so that the two are compiled apart
    const bool has_diag = j1 == t + 1;
    for (int j = 0; ok && j < nt - (has_diag ? 1 : 0); ++j) ok = tile(j, std::false_type{});
    if (ok && has_diag) ok = tile(nt - 1, std::true_type{});
    if (ok && !*abort_flag) ok = warp_wait(o_final, 0, kErrWaitAttention);
    // every softmax thread ends here, so the named barriers below see all 256
    if (!ok) *abort_flag = 1;
    attn_epilogue<D>(p, &tmO, sK, tmem, lane_base, colO, wg, row, grow, h, t, part_code, (t - p.ts) * per_tile + pair, ok,
                     m_run, l_run, 1.0f, abort_flag, &s_last, &s_ready);
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

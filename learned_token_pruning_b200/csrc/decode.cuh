// Decode over the gated KV cache ("TokenGate and T2Quant: a close reading",
// §4.1 Gate module, temperature scaling and engineering notes): one new query
// token attends to every row of the cache, the gate term acting as an
// additive mask on the logits:
//     l_c = temp_h * ratio * sm_scale * (q_h . k_c) + gain_h * bias_c,
//     o_h = sum_c softmax_c(l) v_c
// (bias_c is the kept prompt token's importance and 0 for generated tokens;
// ratio is the step's temperature ratio).  Computed in base 2:
//     x_c = (a_h q_h) . k_c + g_h bias_c,  a_h = temp_h ratio sm_scale log2(e),
//     g_h = gain_h log2(e).
//
// Split-KV: CTA (g, j) takes KV head g and key chunk j and serves every query
// head of g's group, so each cache row is read from memory once.  The work is
// a matrix-vector product per head and is bound by reading the cache, so it
// runs on the CUDA cores:
//   1. the group's query rows, pre-scaled by a_h, into shared memory (fp32);
//   2. logits: four lanes per key, each with a quarter of the head dimension
//      (coalesced 16-byte loads of the key row), reduced over the four lanes;
//   3. the chunk's softmax per head (max, 2^(x - max), sum) in shared memory;
//   4. P V: one output element (head, dimension) per thread, looping over the
//      chunk's keys (the group's heads read the same value row);
//   5. (max, sum, unnormalised O) of the chunk into the workspace; the last CTA
//      of KV head g (a counter) merges the chunks in chunk order, so the
//      result does not depend on which CTA finished when.
#pragma once

#include "attn_tc.cuh"  // packed fp32 pairs (f2_*) and ex2_approx, shared with the attention kernel
#include "common.cuh"
#include "simt.cuh"

namespace tg {

constexpr int kDecThreads = 256;
constexpr int kDecMaxGroup = 8;       // query heads per KV head
constexpr int kDecMaxChunk = 1024;    // keys per CTA
constexpr int kDecMaxChunks = 256;    // chunks per KV head (cache length <= 256 * 1024)
constexpr int kDecKeysPerPass = 64;   // 8 warps x 8 keys

struct DecodeParams {
  const void* q;
  const void* k;
  const void* v;
  int64_t ldk, ldv;
  int length, hq, hkv, group, chunk, nchunks;
  const float* bias;
  const float* gain;
  const float* temp;
  float ratio_scale_log2;  // ratio * sm_scale * log2(e)
  void* out;
  float* lse;
  float* part;         // [hkv][nchunks][group][D + 2]: O, then (max, sum)
  unsigned* counters;  // [hkv], zero on entry
};

// N consecutive elements from 16-byte aligned global memory, as fp32
template <int N>
__device__ __forceinline__ void load_f32(const __nv_bfloat16* src, float (&x)[N]) {
  static_assert(N % 8 == 0, "16-byte vectors of bf16");
#pragma unroll
  for (int i = 0; i < N / 8; ++i) {
    const uint4 w = reinterpret_cast<const uint4*>(src)[i];
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      x[8 * i + 2 * t] = bf16_lo(ww[t]);
      x[8 * i + 2 * t + 1] = bf16_hi(ww[t]);
    }
  }
}
template <int N>
__device__ __forceinline__ void load_f32(const float* src, float (&x)[N]) {
  static_assert(N % 4 == 0, "16-byte vectors of fp32");
#pragma unroll
  for (int i = 0; i < N / 4; ++i) {
    const float4 w = reinterpret_cast<const float4*>(src)[i];
    x[4 * i] = w.x;
    x[4 * i + 1] = w.y;
    x[4 * i + 2] = w.z;
    x[4 * i + 3] = w.w;
  }
}

template <typename T, int D, int GT>
__global__ void __launch_bounds__(kDecThreads) k_decode_attn(DecodeParams p) {
  constexpr int Q4 = D / 4;  // head-dimension elements per lane of a key's four lanes
  // the lane's slice of the group's scaled query rows lives in registers for
  // groups of up to four heads (else it is read from shared memory per key)
  constexpr bool kQReg = GT * Q4 <= 128;
  __shared__ float s_q[kDecMaxGroup][D];
  __shared__ float s_x[kDecMaxGroup][kDecMaxChunk];
  __shared__ float s_red[kDecMaxGroup][kDecThreads / 32];
  __shared__ float s_stat[kDecMaxGroup][2];
  __shared__ float s_pv[kDecThreads * 8];  // P V per key slice: [S][G * D], S * G * D <= 256 * (16 / sizeof(T))
  __shared__ int s_last;
  pdl_wait();
  pdl_launch_dependents();
  const int g = blockIdx.x / p.nchunks, j = blockIdx.x % p.nchunks;
  const int c0 = j * p.chunk, c1 = min(c0 + p.chunk, p.length), nk = c1 - c0;
  constexpr int G = GT;
  const int h0 = g * G;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const T* qp = static_cast<const T*>(p.q);
  const T* kp = static_cast<const T*>(p.k);
  const T* vp = static_cast<const T*>(p.v);

  // 1. scaled query rows
  for (int i = threadIdx.x; i < G * D; i += kDecThreads) {
    const int u = i / D, d = i % D;
    s_q[u][d] = to_f32(qp[static_cast<int64_t>(h0 + u) * D + d]) * (p.temp[h0 + u] * p.ratio_scale_log2);
  }
  __syncthreads();

  // 2. logits of the chunk's keys: key = pass base + warp * 8 + lane / 4, quarter = lane % 4
  const int qd = (lane & 3) * Q4;
  float qreg[kQReg ? G : 1][kQReg ? Q4 : 1];
  if constexpr (kQReg) {
#pragma unroll
    for (int u = 0; u < G; ++u)
#pragma unroll
      for (int e = 0; e < Q4; ++e) qreg[u][e] = s_q[u][qd + e];
  }
  float gbias[G];
#pragma unroll
  for (int u = 0; u < G; ++u) gbias[u] = p.gain[h0 + u] * kLog2e;
  for (int base = 0; base < nk; base += kDecKeysPerPass) {
    const int kk = base + warp * 8 + (lane >> 2);
    float acc[G];
#pragma unroll
    for (int u = 0; u < G; ++u) acc[u] = 0.0f;
    if (kk < nk) {
      float kv[Q4];
      load_f32<Q4>(kp + static_cast<int64_t>(c0 + kk) * p.ldk + static_cast<int64_t>(g) * D + qd, kv);
#pragma unroll
      for (int e = 0; e < Q4; ++e) {
#pragma unroll
        for (int u = 0; u < G; ++u) acc[u] = fmaf(kQReg ? qreg[kQReg ? u : 0][kQReg ? e : 0] : s_q[u][qd + e], kv[e], acc[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < G; ++u) {
      acc[u] += __shfl_xor_sync(0xffffffffu, acc[u], 1);
      acc[u] += __shfl_xor_sync(0xffffffffu, acc[u], 2);
    }
    if (kk < nk && (lane & 3) == 0) {
      const float b = p.bias ? p.bias[c0 + kk] : 0.0f;
#pragma unroll
      for (int u = 0; u < G; ++u) s_x[u][kk] = fmaf(gbias[u], b, acc[u]);
    }
  }
  __syncthreads();

  // 3. softmax of the chunk per head: max, then p = 2^(x - max) in place, then the sum
  for (int u = 0; u < G; ++u) {
    float mx = -INFINITY;
    for (int c = threadIdx.x; c < nk; c += kDecThreads) mx = fmaxf(mx, s_x[u][c]);
#pragma unroll
    for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) s_red[u][warp] = mx;
  }
  __syncthreads();
  if (threadIdx.x < G) {
    float mx = -INFINITY;
    for (int w = 0; w < kDecThreads / 32; ++w) mx = fmaxf(mx, s_red[threadIdx.x][w]);
    s_stat[threadIdx.x][0] = mx;
  }
  __syncthreads();
  for (int u = 0; u < G; ++u) {
    const float mx = s_stat[u][0];
    float sum = 0.0f;
    for (int c = threadIdx.x; c < nk; c += kDecThreads) {
      const float e = exp2f(s_x[u][c] - mx);
      s_x[u][c] = e;
      sum += e;
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane == 0) s_red[u][warp] = sum;
  }
  __syncthreads();
  if (threadIdx.x < G) {
    float sum = 0.0f;
    for (int w = 0; w < kDecThreads / 32; ++w) sum += s_red[threadIdx.x][w];
    s_stat[threadIdx.x][1] = sum;
  }

  // 4. unnormalised O = P V of the chunk.  Thread -> (key slice, head u,
  //    16-byte group of VW dimensions): each reads value rows c = slice,
  //    slice + S, ... with one vector load per row; the S slices are added in
  //    slice order through shared memory.
  constexpr int VW = 16 / sizeof(T);
  constexpr int DV = D / VW;
  const int groups = G * DV;
  const int S = kDecThreads / groups;
  if (threadIdx.x < S * groups) {
    const int slice = threadIdx.x / groups, rem = threadIdx.x % groups, u = rem / DV, dv = rem % DV;
    const T* vbase = vp + static_cast<int64_t>(c0) * p.ldv + static_cast<int64_t>(g) * D + dv * VW;
    float acc[VW];
#pragma unroll
    for (int e = 0; e < VW; ++e) acc[e] = 0.0f;
    int c = slice;
    for (; c + 3 * S < nk; c += 4 * S) {  // four rows in flight
      float vv[4][VW];
#pragma unroll
      for (int r = 0; r < 4; ++r) load_f32<VW>(vbase + static_cast<int64_t>(c + r * S) * p.ldv, vv[r]);
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const float pc = s_x[u][c + r * S];
#pragma unroll
        for (int e = 0; e < VW; ++e) acc[e] = fmaf(pc, vv[r][e], acc[e]);
      }
    }
    for (; c < nk; c += S) {
      float vv[VW];
      load_f32<VW>(vbase + static_cast<int64_t>(c) * p.ldv, vv);
      const float pc = s_x[u][c];
#pragma unroll
      for (int e = 0; e < VW; ++e) acc[e] = fmaf(pc, vv[e], acc[e]);
    }
#pragma unroll
    for (int e = 0; e < VW; ++e) s_pv[slice * (G * D) + u * D + dv * VW + e] = acc[e];
  }
  __syncthreads();  // every slice's sums and s_stat of every head are written
  float* part = p.part + (static_cast<size_t>(g) * p.nchunks + j) * G * (D + 2);
  for (int i = threadIdx.x; i < G * D; i += kDecThreads) {
    float o = 0.0f;
    for (int sl = 0; sl < S; ++sl) o += s_pv[sl * (G * D) + i];
    part[(i / D) * (D + 2) + (i % D)] = o;
  }
  if (threadIdx.x < G) {
    part[threadIdx.x * (D + 2) + D] = s_stat[threadIdx.x][0];
    part[threadIdx.x * (D + 2) + D + 1] = s_stat[threadIdx.x][1];
  }

  // 5. the last CTA of KV head g merges the chunks in chunk order
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = atomicAdd(&p.counters[g], 1u) == static_cast<unsigned>(p.nchunks - 1) ? 1 : 0;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const int nc = p.nchunks;
  const float* gpart = p.part + static_cast<size_t>(g) * nc * G * (D + 2);
  float* s_m = &s_x[0][0];                     // [G][nc] chunk maxima, then weights
  float* s_l = &s_x[0][0] + kDecMaxGroup * kDecMaxChunks;  // [G][nc] chunk sums
  for (int i = threadIdx.x; i < G * nc; i += kDecThreads) {
    const int u = i / nc, jj = i % nc;
    s_m[i] = __ldcg(gpart + (jj * G + u) * (D + 2) + D);
    s_l[i] = __ldcg(gpart + (jj * G + u) * (D + 2) + D + 1);
  }
  __syncthreads();
  if (threadIdx.x < G) {
    // per head: the overall maximum, each chunk's weight 2^(m_j - max), the
    // total sum; the weights (divided by the sum) replace the maxima
    const int u = threadIdx.x;
    float mx = -INFINITY;
    for (int jj = 0; jj < nc; ++jj) mx = fmaxf(mx, s_m[u * nc + jj]);
    float l = 0.0f;
    for (int jj = 0; jj < nc; ++jj) {
      const float w = exp2f(s_m[u * nc + jj] - mx);
      s_m[u * nc + jj] = w;
      l = fmaf(s_l[u * nc + jj], w, l);
    }
    const float inv = 1.0f / l;
    for (int jj = 0; jj < nc; ++jj) s_m[u * nc + jj] *= inv;
    if (p.lse) p.lse[h0 + u] = (mx + log2f(l)) * kLn2;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < G * D; i += kDecThreads) {
    const int u = i / D, d = i % D;
    const float* po = gpart + u * (D + 2) + d;
    float o0 = 0.0f, o1 = 0.0f, o2 = 0.0f, o3 = 0.0f;
    int jj = 0;
    for (; jj + 4 <= nc; jj += 4) {
      o0 = fmaf(s_m[u * nc + jj], __ldcg(po + (jj + 0) * G * (D + 2)), o0);
      o1 = fmaf(s_m[u * nc + jj + 1], __ldcg(po + (jj + 1) * G * (D + 2)), o1);
      o2 = fmaf(s_m[u * nc + jj + 2], __ldcg(po + (jj + 2) * G * (D + 2)), o2);
      o3 = fmaf(s_m[u * nc + jj + 3], __ldcg(po + (jj + 3) * G * (D + 2)), o3);
    }
    for (; jj < nc; ++jj) o0 = fmaf(s_m[u * nc + jj], __ldcg(po + jj * G * (D + 2)), o0);
    static_cast<T*>(p.out)[static_cast<int64_t>(h0 + u) * D + d] = from_f32<T>((o0 + o1) + (o2 + o3));
  }
  if (threadIdx.x == 0) p.counters[g] = 0u;  // ready for the next call
}


// ---------------------------------------------------------------------------
// bf16 cache: the same computation with the cache rows streamed through
// shared memory by TMA, so the bytes in flight no longer depend on registers
// or on the phase the warps are in.  CTA (g, j) takes KV head g and a chunk of
// rows (one wave: about one CTA per SM over all KV heads).  Warp 8 loads
// 64-row tiles of K and V (128-byte swizzled boxes of 64 head dimensions),
// and the tile's 64 key biases, into a ring of 128 KB (a bias read by the
// threads themselves one tile ahead would wait on DRAM under the full load);
// warps 0-7 take each tile in two steps:
//   logits: four lanes per key, lane qq holding 16-byte chunks qq, qq + 4, ...
//     of the key row (the swizzle spreads a warp's eight keys over all banks);
//   P V: thread (key slice, head, 16-byte group of dimensions) keeps an
//     online softmax over its own slice of the keys (running maximum M and
//     sum l; the tile's slice maximum, the rescale factor 2^(M_old - M),
//     p = 2^(x - M)) and adds p v of the slice's rows of the tile.
// One named barrier per tile (logits before P V).  At the end the slices are
// rescaled to the largest slice maximum and added in slice order, and (M, l,
// O) of the chunk go to the same workspace layout and chunk-order merge as
// above.
// Two fp32 fused multiply-adds in one instruction on float2 values
// (fma.rn.f32x2): per lane exactly fmaf(a, b, c).
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  f2_unpack(f2_fma(f2_pack(a.x, a.y), f2_pack(b.x, b.y), f2_pack(c.x, c.y)), d.x, d.y);
  return d;
}

constexpr int kDtRows = 64;        // cache rows per tile
constexpr int kDtThreads = 288;    // 8 compute warps + 1 producer warp
constexpr int kDtCompute = 256;
constexpr int kDtRingBytes = 128 * 1024;

template <int D>
struct DecTmaCfg {
  static constexpr int kBoxes = D / 64;                      // 64-dimension boxes per row
  static constexpr int kBoxBytes = kDtRows * 128;
  static constexpr int kTileBytes = kBoxes * kBoxBytes;      // K or V tile
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kStages = kDtRingBytes / kStageBytes;  // 4 (D = 128) or 8 (D = 64)
  static constexpr size_t kFloats = static_cast<size_t>(kDecMaxGroup) * D      // s_q
                                    + 2 * kDecMaxGroup * kDtRows               // s_x, two tiles
                                    + 64                                       // s_ml
                                    + kDtCompute * 8                           // s_pv
                                    + 2 * kDecMaxGroup * kDecMaxChunks;        // merge
  static constexpr int kBiasBytes = kDtRows * 4;            // the tile's key biases
  static constexpr size_t kSmem = 1024 + kDtRingBytes + kStages * kBiasBytes + kFloats * 4 + 2 * kStages * 8;
};

template <int D, int G>
__global__ void __launch_bounds__(kDtThreads, 1)
    k_decode_tma(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                 const __grid_constant__ CUtensorMap tmBias, DecodeParams p) {
  using Cfg = DecTmaCfg<D>;
  constexpr int R = kDtRows, S = Cfg::kStages;
  extern __shared__ uint8_t dec_smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dec_smem_raw) + 1023) & ~uintptr_t(1023));
  float* s_bias = reinterpret_cast<float*>(ring + kDtRingBytes);  // [S][R] key biases per stage
  float* s_q = s_bias + S * R;                                 // [G][D] query rows scaled by a_h
  float* s_x = s_q + kDecMaxGroup * D;                         // [2][G][R] logits, then p, per tile parity
  float* s_ml = s_x + 2 * kDecMaxGroup * R;                    // [slices][G][2] (M, l) per slice and head
  float* s_pv = s_ml + 64;                                     // [slices][G * D]
  float* s_merge = s_pv + kDtCompute * 8;                      // [2][G][nchunks]
  uint64_t* full = reinterpret_cast<uint64_t*>(s_merge + 2 * kDecMaxGroup * kDecMaxChunks);
  uint64_t* empty = full + S;
  __shared__ int s_last;
  // [tile parity] a compute warp's wait for tile t ran out: set before tile
  // t's named barrier and read by every compute warp right after it (a set
  // for tile t + 2 needs every warp past tile t + 1's barrier), so all of
  // them leave at the same tile
  __shared__ volatile int s_stop[2];
  __shared__ volatile int s_pstop;  // the producer's wait ran out

  const int g = blockIdx.x / p.nchunks, j = blockIdx.x % p.nchunks;
  const int c0 = j * p.chunk, c1 = min(c0 + p.chunk, p.length), nk = c1 - c0;
  const int ntiles = (nk + R - 1) / R;
  const int h0 = g * G;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kDtCompute / 32);
    }
    s_stop[0] = s_stop[1] = 0;
    s_pstop = 0;
    fence_mbar_init();
  }
  pdl_wait();
  pdl_launch_dependents();
  const __nv_bfloat16* qp = static_cast<const __nv_bfloat16*>(p.q);
  for (int i = threadIdx.x; i < G * D; i += kDtThreads) {
    const int u = i / D, d = i % D;
    s_q[i] = __bfloat162float(qp[static_cast<int64_t>(h0 + u) * D + d]) * (p.temp[h0 + u] * p.ratio_scale_log2);
  }
  __syncthreads();

  // P V mapping: PAIRS (head, 16-byte dimension group) per slice, SL slices
  constexpr int DG = D / 8;
  constexpr int PAIRS = G * DG;
  constexpr int SL = kDtCompute / PAIRS;
  float2 acc[4];  // dimensions 8 pdg + 2h, 8 pdg + 2h + 1
#pragma unroll
  for (int h = 0; h < 4; ++h) acc[h] = make_float2(0.0f, 0.0f);
  const int pair = threadIdx.x % PAIRS, slice = threadIdx.x / PAIRS;
  const int pu = pair / DG, pdg = pair % DG;
  float m_run = -INFINITY, l_run = 0.0f;  // running maximum and sum of this thread's key slice and head

  if (warp == kDtCompute / 32) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      if (p.bias) prefetch_tmap(&tmBias);
      for (int t = 0; t < ntiles; ++t) {
        const int st = t % S;
        if (!mbar_wait(&empty[st], ((t / S) & 1) ^ 1, kErrWaitAttention)) {
          s_pstop = 1;
          break;
        }
        mbar_arrive_expect_tx(&full[st], Cfg::kStageBytes + (p.bias ? Cfg::kBiasBytes : 0));
        uint8_t* dst = ring + st * Cfg::kStageBytes;
        const int y = c0 + t * R;  // rows past the cache read as zeros
        if (p.bias) tma_load_1d(s_bias + st * R, &tmBias, &full[st], y);
#pragma unroll
        for (int b = 0; b < Cfg::kBoxes; ++b) {
          tma_load_2d(dst + b * Cfg::kBoxBytes, &tmK, &full[st], g * D + b * 64, y);
          tma_load_2d(dst + Cfg::kTileBytes + b * Cfg::kBoxBytes, &tmV, &full[st], g * D + b * 64, y);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ compute warps
    constexpr int NM = D / 32;  // 16-byte chunks per lane per key
    constexpr bool kQReg = G * D / 4 <= 64;
    const int kr = threadIdx.x >> 2, qq = threadIdx.x & 3;
    float qreg[kQReg ? G : 1][kQReg ? D / 4 : 1];
    if constexpr (kQReg) {
#pragma unroll
      for (int u = 0; u < G; ++u)
#pragma unroll
        for (int m = 0; m < NM; ++m)
#pragma unroll
          for (int e = 0; e < 8; ++e) qreg[u][m * 8 + e] = s_q[u * D + 8 * (qq + 4 * m) + e];
    }
    float gbias[G];
#pragma unroll
    for (int u = 0; u < G; ++u) gbias[u] = p.gain[h0 + u] * kLog2e;
    for (int t = 0; t < ntiles; ++t) {
      const int st = t % S;
      const bool ok = warp_wait(&full[st], (t / S) & 1, kErrWaitAttention);
      if (!ok && lane == 0) s_stop[t & 1] = 1;
      const uint8_t* kt = ring + st * Cfg::kStageBytes;
      float* sx = s_x + (t & 1) * (kDecMaxGroup * R);
      // logits (per head an fp32 pair of partial sums over even and odd dimensions)
      float2 xa2[G];
#pragma unroll
      for (int u = 0; u < G; ++u) xa2[u] = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int m = 0; m < NM; ++m) {
        const int c = qq + 4 * m;
        const uint4 w = *reinterpret_cast<const uint4*>(kt + (c >> 3) * Cfg::kBoxBytes + kr * 128 +
                                                        (((c & 7) ^ (kr & 7)) << 4));
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const float k0 = bf16_lo(ww[h]), k1 = bf16_hi(ww[h]);
#pragma unroll
          for (int u = 0; u < G; ++u) {
            const float q0 = kQReg ? qreg[kQReg ? u : 0][kQReg ? m * 8 + 2 * h : 0] : s_q[u * D + 8 * c + 2 * h];
            const float q1 = kQReg ? qreg[kQReg ? u : 0][kQReg ? m * 8 + 2 * h + 1 : 0] : s_q[u * D + 8 * c + 2 * h + 1];
            xa2[u] = ffma2(make_float2(q0, q1), make_float2(k0, k1), xa2[u]);
          }
        }
      }
      float xa[G];
#pragma unroll
      for (int u = 0; u < G; ++u) {
        xa[u] = xa2[u].x + xa2[u].y;
        xa[u] += __shfl_xor_sync(0xffffffffu, xa[u], 1);
        xa[u] += __shfl_xor_sync(0xffffffffu, xa[u], 2);
      }
      const int key = t * R + kr;
      if (qq == 0) {
        const float b = p.bias ? s_bias[st * R + kr] : 0.0f;
#pragma unroll
        for (int u = 0; u < G; ++u) sx[u * R + kr] = key < nk ? fmaf(gbias[u], b, xa[u]) : -INFINITY;
      }
      asm volatile("bar.sync 1, 256;" ::: "memory");
      if (s_stop[t & 1]) break;
      // P V, each thread with its own online softmax over its slice of the
      // keys (running maximum M and sum l per slice and head, no barrier
      // between the two steps; the slices are merged like chunks at the end)
      if (slice < SL) {
        const float* xx = sx + pu * R;
        float tmax = -INFINITY;
#pragma unroll 4
        for (int c = slice; c < R; c += SL) tmax = fmaxf(tmax, xx[c]);
        const float m_new = fmaxf(m_run, tmax);
        const float m_use = m_new == -INFINITY ? 0.0f : m_new;  // no key of the slice yet: all weights 0
        const float alpha = ex2_approx(m_run - m_use);
        m_run = m_new;
        l_run *= alpha;
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          acc[h].x *= alpha;
          acc[h].y *= alpha;
        }
        const uint8_t* vt = kt + Cfg::kTileBytes + (pdg >> 3) * Cfg::kBoxBytes;
#pragma unroll 4
        for (int c = slice; c < R; c += SL) {
          const float pc = ex2_approx(xx[c] - m_use);
          l_run += pc;
          const uint4 w = *reinterpret_cast<const uint4*>(vt + c * 128 + (((pdg & 7) ^ (c & 7)) << 4));
          const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int h = 0; h < 4; ++h) acc[h] = ffma2(make_float2(pc, pc), make_float2(bf16_lo(ww[h]), bf16_hi(ww[h])), acc[h]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);  // this warp's reads of the stage are done
    }
    if (!(s_stop[0] | s_stop[1]) && slice < SL) {
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        s_pv[slice * (G * D) + pu * D + pdg * 8 + 2 * h] = acc[h].x;
        s_pv[slice * (G * D) + pu * D + pdg * 8 + 2 * h + 1] = acc[h].y;
      }
      if (pdg == 0) {
        s_ml[(slice * G + pu) * 2] = m_run;
        s_ml[(slice * G + pu) * 2 + 1] = l_run;
      }
    }
  }
  __syncthreads();
  if (s_stop[0] | s_stop[1] | s_pstop) return;  // a wait ran out (recorded in the error word)

  // the chunk's (M, l, unnormalised O): the slices rescaled to the largest
  // slice maximum and added in slice order
  float* part = p.part + (static_cast<size_t>(g) * p.nchunks + j) * G * (D + 2);
  for (int i = threadIdx.x; i < G * D; i += kDtThreads) {
    const int u = i / D;
    float mx = -INFINITY;
    for (int sl = 0; sl < SL; ++sl) mx = fmaxf(mx, s_ml[(sl * G + u) * 2]);
    float o = 0.0f;
    for (int sl = 0; sl < SL; ++sl) o = fmaf(exp2f(s_ml[(sl * G + u) * 2] - mx), s_pv[sl * (G * D) + i], o);
    part[u * (D + 2) + (i % D)] = o;
  }
  if (threadIdx.x < G) {
    const int u = threadIdx.x;
    float mx = -INFINITY;
    for (int sl = 0; sl < SL; ++sl) mx = fmaxf(mx, s_ml[(sl * G + u) * 2]);
    float l = 0.0f;
    for (int sl = 0; sl < SL; ++sl) l = fmaf(exp2f(s_ml[(sl * G + u) * 2] - mx), s_ml[(sl * G + u) * 2 + 1], l);
    part[u * (D + 2) + D] = mx;
    part[u * (D + 2) + D + 1] = l;
  }

  // the last CTA of KV head g merges the chunks in chunk order
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = atomicAdd(&p.counters[g], 1u) == static_cast<unsigned>(p.nchunks - 1) ? 1 : 0;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const int nc = p.nchunks;
  const float* gpart = p.part + static_cast<size_t>(g) * nc * G * (D + 2);
  float* s_m = s_merge;                 // [G][nc] chunk maxima, then weights
  float* s_l = s_merge + G * nc;        // [G][nc] chunk sums
  for (int i = threadIdx.x; i < G * nc; i += kDtThreads) {
    const int u = i / nc, jj = i % nc;
    s_m[i] = __ldcg(gpart + (jj * G + u) * (D + 2) + D);
    s_l[i] = __ldcg(gpart + (jj * G + u) * (D + 2) + D + 1);
  }
  __syncthreads();
  if (threadIdx.x < G) {
    const int u = threadIdx.x;
    float mx = -INFINITY;
    for (int jj = 0; jj < nc; ++jj) mx = fmaxf(mx, s_m[u * nc + jj]);
    float l = 0.0f;
    for (int jj = 0; jj < nc; ++jj) {
      const float w = exp2f(s_m[u * nc + jj] - mx);
      s_m[u * nc + jj] = w;
      l = fmaf(s_l[u * nc + jj], w, l);
    }
    const float inv = 1.0f / l;
    for (int jj = 0; jj < nc; ++jj) s_m[u * nc + jj] *= inv;
    if (p.lse) p.lse[h0 + u] = (mx + log2f(l)) * kLn2;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < G * D; i += kDtThreads) {
    const int u = i / D, d = i % D;
    const float* po = gpart + u * (D + 2) + d;
    float o0 = 0.0f, o1 = 0.0f;
    int jj = 0;
    for (; jj + 2 <= nc; jj += 2) {
      o0 = fmaf(s_m[u * nc + jj], __ldcg(po + jj * G * (D + 2)), o0);
      o1 = fmaf(s_m[u * nc + jj + 1], __ldcg(po + (jj + 1) * G * (D + 2)), o1);
    }
    for (; jj < nc; ++jj) o0 = fmaf(s_m[u * nc + jj], __ldcg(po + jj * G * (D + 2)), o0);
    static_cast<__nv_bfloat16*>(p.out)[static_cast<int64_t>(h0 + u) * D + d] = from_f32<__nv_bfloat16>(o0 + o1);
  }
  if (threadIdx.x == 0) p.counters[g] = 0u;  // ready for the next call
}

}  // namespace tg

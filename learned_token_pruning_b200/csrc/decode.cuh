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

}  // namespace tg

// CUDA-core kernels: the fp32 path of every op (the tensor cores have no
// exact-fp32 mode), the row-wise pieces of the decoder layer (RMSNorm, q/k
// norm + RoPE, SwiGLU) and the shapes the tensor-core kernels do not take.
#pragma once

#include "common.cuh"

namespace tg {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// ---------------------------------------------------------------------------
// Gate scores on CUDA cores: one warp per token.
// "TokenGate and T2Quant: a close reading", §4.1 Gate module:
//   s_j = w2 . SiLU(W1 RMSNorm(h_j) + b1) + b2 for prunable j, else 0.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256) k_gate_score_simt(const T* __restrict__ hidden, int64_t n, int d,
                                                         const float* __restrict__ norm_w, float eps,
                                                         const T* __restrict__ w1, const float* __restrict__ b1,
                                                         const float* __restrict__ w2, float b2, int h,
                                                         const uint8_t* __restrict__ prunable,
                                                         float* __restrict__ scores) {
  const int lane = threadIdx.x & 31;
  const int64_t j = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (j >= n) return;
  const T* row = hidden + j * d;
  if (prunable[j] == 0) {
    if (lane == 0) scores[j] = 0.0f;
    return;
  }
  float ss = 0.0f;
  for (int i = lane; i < d; i += 32) {
    const float x = to_f32(row[i]);
    ss += x * x;
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float inv = 1.0f / sqrtf(ss / static_cast<float>(d) + eps);
  float s = 0.0f;
  for (int u = 0; u < h; ++u) {
    const T* wr = w1 + static_cast<int64_t>(u) * d;
    float acc = 0.0f;
    for (int i = lane; i < d; i += 32) {
      const float x = to_f32(row[i]) * (norm_w ? norm_w[i] : 1.0f);
      acc += x * to_f32(wr[i]);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    const float v = acc * inv + (b1 ? b1[u] : 0.0f);
    s += w2[u] * (v / (1.0f + expf(-v)));
  }
  if (lane == 0) scores[j] = s + b2;
}

// w1f[u][i] = w1[u][i] * norm_w[i], rounded to bf16 (the norm weight folded into the gate's first layer)
__global__ void __launch_bounds__(256) k_fold_norm(const __nv_bfloat16* __restrict__ w1, const float* __restrict__ nw,
                                                   __nv_bfloat16* __restrict__ w1f, int64_t total, int d) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
  if (i < total) w1f[i] = __float2bfloat16_rn(__bfloat162float(w1[i]) * nw[i % d]);
}

// sumsq = sum over prunable j of s_j^2, one block, fixed summation order.
__global__ void __launch_bounds__(1024) k_sumsq_ordered(const float* __restrict__ scores,
                                                        const uint8_t* __restrict__ prunable, int64_t n,
                                                        float* __restrict__ sumsq) {
  __shared__ float part[32];
  float acc = 0.0f;
  for (int64_t j = threadIdx.x; j < n; j += blockDim.x) {
    const float s = scores[j];
    if (prunable[j]) acc += s * s;
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < (blockDim.x >> 5) ? part[threadIdx.x] : 0.0f;
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (threadIdx.x == 0) sumsq[0] = v;
  }
}

// ---------------------------------------------------------------------------
// Token-gated causal GQA attention on CUDA cores (fp32 accumulate).
// Block: 16 query rows of one head, 8 threads per row; each thread owns the
// head dims e*8 + sub.  Keys stream through shared memory in tiles of 32.
//   l_rc = temp_h * ratio_r * sm_scale * (q_r . k_c) + gain_h * bias_c ; online softmax in base 2.
// ---------------------------------------------------------------------------
struct AttnSimtParams {
  const void* q;
  const void* k;
  const void* v;
  int64_t ldq, ldk, ldv, ldo;
  int m, hq, hkv;
  const float* bias;
  const float* gain;
  const float* temp;
  const float* ratio;
  float sm_scale;
  void* out;
  float* lse;
};

template <typename T, int D>
__global__ void __launch_bounds__(128) k_attn_simt(AttnSimtParams p) {
  constexpr int E = D / 8;
  constexpr int KT = 32;
  __shared__ float sk[KT][D];
  __shared__ float sv[KT][D];
  __shared__ float sb[KT];
  const T* Q = static_cast<const T*>(p.q);
  const T* Kp = static_cast<const T*>(p.k);
  const T* Vp = static_cast<const T*>(p.v);
  const int h = blockIdx.y;
  const int g = h / (p.hq / p.hkv);
  const int row_in = threadIdx.x >> 3, sub = threadIdx.x & 7;
  const int r = blockIdx.x * 16 + row_in;
  const bool valid = r < p.m;
  const float a_row =
      valid ? p.temp[h] * (p.ratio ? p.ratio[r] : 1.0f) * p.sm_scale * kLog2e : 0.0f;
  const float gb = p.gain[h] * kLog2e;
  float q[E], o[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    q[e] = valid ? to_f32(Q[static_cast<int64_t>(r) * p.ldq + h * D + e * 8 + sub]) : 0.0f;
    o[e] = 0.0f;
  }
  float mrun = -INFINITY, lrun = 0.0f;
  const int last_row = min(p.m - 1, blockIdx.x * 16 + 15);
  for (int c0 = 0; c0 <= last_row; c0 += KT) {
    __syncthreads();
    for (int t = threadIdx.x; t < KT * D; t += 128) {
      const int cc = t / D, dd = t - cc * D;
      const int c = c0 + cc;
      float kv = 0.0f, vv = 0.0f;
      if (c < p.m) {
        kv = to_f32(Kp[static_cast<int64_t>(c) * p.ldk + g * D + dd]);
        vv = to_f32(Vp[static_cast<int64_t>(c) * p.ldv + g * D + dd]);
      }
      sk[cc][dd] = kv;
      sv[cc][dd] = vv;
    }
    if (threadIdx.x < KT) {
      const int c = c0 + threadIdx.x;
      sb[threadIdx.x] = (c < p.m && p.bias) ? gb * p.bias[c] : 0.0f;
    }
    __syncthreads();
    const int cmax = min(KT, r - c0 + 1);  // keys c0 .. r are visible
    for (int cc = 0; cc < KT; ++cc) {
      float part = 0.0f;
#pragma unroll
      for (int e = 0; e < E; ++e) part += q[e] * sk[cc][e * 8 + sub];
      part += __shfl_xor_sync(0xffffffffu, part, 1);
      part += __shfl_xor_sync(0xffffffffu, part, 2);
      part += __shfl_xor_sync(0xffffffffu, part, 4);
      if (cc < cmax) {
        const float x = a_row * part + sb[cc];
        const float mnew = fmaxf(mrun, x);
        const float sc = exp2f(mrun - mnew);
        const float pr = exp2f(x - mnew);
        lrun = lrun * sc + pr;
#pragma unroll
        for (int e = 0; e < E; ++e) o[e] = o[e] * sc + pr * sv[cc][e * 8 + sub];
        mrun = mnew;
      }
    }
  }
  if (valid) {
    T* O = static_cast<T*>(p.out);
    const float inv = 1.0f / lrun;
#pragma unroll
    for (int e = 0; e < E; ++e) O[static_cast<int64_t>(r) * p.ldo + h * D + e * 8 + sub] = from_f32<T>(o[e] * inv);
    if (p.lse && sub == 0) p.lse[static_cast<int64_t>(h) * p.m + r] = (mrun + log2f(lrun)) * kLn2;
  }
}

// ---------------------------------------------------------------------------
// C = A B^T (+ C) on CUDA cores; A [M][K] (lda), B [N][K], C [M][N] (ldc).
// 64x64 tiles, 16-deep k slices, 4x4 outputs per thread, fp32 accumulation.
// ---------------------------------------------------------------------------
template <typename T, bool kResidual>
__global__ void __launch_bounds__(256) k_gemm_simt(const T* __restrict__ A, int64_t lda, const T* __restrict__ B,
                                                   T* __restrict__ C, int64_t ldc, int M, int N, int K) {
  __shared__ float As[16][64 + 4];
  __shared__ float Bs[16][64 + 4];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += 16) {
    for (int t = threadIdx.x; t < 64 * 16; t += 256) {
      const int rr = t >> 4, kk = t & 15;
      const int gm = m0 + rr, gn = n0 + rr, gk = k0 + kk;
      As[kk][rr] = (gm < M && gk < K) ? to_f32(A[static_cast<int64_t>(gm) * lda + gk]) : 0.0f;
      Bs[kk][rr] = (gn < N && gk < K) ? to_f32(B[static_cast<int64_t>(gn) * K + gk]) : 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = As[kk][ty * 4 + i];
        b[i] = Bs[kk][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) acc[i][jj] += a[i] * b[jj];
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int gm = m0 + ty * 4 + i;
    if (gm >= M) continue;
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      const int gn = n0 + tx * 4 + jj;
      if (gn >= N) continue;
      T* c = C + static_cast<int64_t>(gm) * ldc + gn;
      float v = acc[i][jj];
      if (kResidual) v += to_f32(*c);
      *c = from_f32<T>(v);
    }
  }
}

// ---------------------------------------------------------------------------
// Row RMSNorm: y = x / sqrt(mean(x^2) + eps) * w; one block per row, 16-byte
// vector accesses (the row is read twice; the second read hits L1).
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256) k_rmsnorm(const T* __restrict__ x, T* __restrict__ y,
                                                 const float* __restrict__ w, int d, float eps) {
  pdl_wait();
  pdl_launch_dependents();
  constexpr int V = 16 / sizeof(T);  // elements per 16-byte vector
  __shared__ float part[8];
  const T* xr = x + static_cast<int64_t>(blockIdx.x) * d;
  T* yr = y + static_cast<int64_t>(blockIdx.x) * d;
  const int nv = d / V;  // d % V == 0 (checked by the caller)
  float ss = 0.0f;
  for (int c = threadIdx.x; c < nv; c += 256) {
    const uint4 v = reinterpret_cast<const uint4*>(xr)[c];
    const T* e = reinterpret_cast<const T*>(&v);
#pragma unroll
    for (int t = 0; t < V; ++t) {
      const float f = to_f32(e[t]);
      ss = fmaf(f, f, ss);
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) tot += part[i];
  const float inv = 1.0f / sqrtf(tot / static_cast<float>(d) + eps);
  for (int c = threadIdx.x; c < nv; c += 256) {
    const uint4 v = reinterpret_cast<const uint4*>(xr)[c];
    const T* e = reinterpret_cast<const T*>(&v);
    uint4 o;
    T* oe = reinterpret_cast<T*>(&o);
#pragma unroll
    for (int t = 0; t < V; ++t) oe[t] = from_f32<T>(to_f32(e[t]) * inv * (w ? w[c * V + t] : 1.0f));
    reinterpret_cast<uint4*>(yr)[c] = o;
  }
}

// ---------------------------------------------------------------------------
// Per-head q/k RMSNorm (optional) and rotate-half RoPE at the original token
// positions, in place on the fused qkv rows.  A block takes 256/(D/2) rows:
// first one thread per (row, frequency) forms cos/sin of pos * theta^(-2i/D)
// in double precision (positions reach 2^17) into shared memory, then each
// warp walks the (row, head) items of the hq + hkv rotated heads; lane l holds
// dims l*E .. l*E+E-1 of the first half and the matching dims of the second.
// ---------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(256) k_qk_norm_rope(T* __restrict__ qkv, int64_t ld, int m, int hq, int hkv,
                                                      const int32_t* __restrict__ pos,
                                                      const float* __restrict__ wq, const float* __restrict__ wk,
                                                      int qk_norm, float eps, float theta) {
  constexpr int H2 = D / 2;
  constexpr int E = H2 / 32;
  constexpr int ROWS = 256 / H2;
  __shared__ float2 cs[ROWS][H2];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int r0 = blockIdx.x * ROWS;
  {
    const int rr = threadIdx.x / H2, i = threadIdx.x % H2;
    const int r = r0 + rr;
    float2 v = make_float2(1.0f, 0.0f);
    if (r < m) {
      const double p = static_cast<double>(pos ? pos[r] : r);
      const double ang = p * exp(-2.0 * static_cast<double>(i) / static_cast<double>(D) * log(static_cast<double>(theta)));
      double sn, cn;
      sincos(ang, &sn, &cn);
      v = make_float2(static_cast<float>(cn), static_cast<float>(sn));
    }
    cs[rr][i] = v;
  }
  __syncthreads();
  const int heads = hq + hkv;
  for (int item = warp; item < ROWS * heads; item += 8) {
    const int rr = item / heads, hh = item - rr * heads;
    const int r = r0 + rr;
    if (r >= m) continue;  // warp-uniform
    T* x = qkv + static_cast<int64_t>(r) * ld + static_cast<int64_t>(hh) * D;
    float a[E], b[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
      a[e] = to_f32(x[lane * E + e]);
      b[e] = to_f32(x[H2 + lane * E + e]);
    }
    if (qk_norm) {
      float ss = 0.0f;
#pragma unroll
      for (int e = 0; e < E; ++e) ss += a[e] * a[e] + b[e] * b[e];
#pragma unroll
      for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      const float inv = 1.0f / sqrtf(ss / static_cast<float>(D) + eps);
      const float* w = hh < hq ? wq : wk;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        a[e] *= inv * w[lane * E + e];
        b[e] *= inv * w[H2 + lane * E + e];
      }
    }
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const float2 c = cs[rr][lane * E + e];
      x[lane * E + e] = from_f32<T>(a[e] * c.x - b[e] * c.y);
      x[H2 + lane * E + e] = from_f32<T>(b[e] * c.x + a[e] * c.y);
    }
  }
}

// ---------------------------------------------------------------------------
// RMSNorm with one warp per row (eight rows per block): the row stays in
// registers between the sum of squares and the scaling, so it is read once,
// and all of a lane's 16-byte loads are in flight together.  MAXV bounds the
// vectors per lane (d <= 32 * MAXV * 16 / sizeof(T)); w, if given, is
// 16-byte aligned.
// ---------------------------------------------------------------------------
template <typename T, int MAXV>
__global__ void __launch_bounds__(256) k_rmsnorm_warp(const T* __restrict__ x, T* __restrict__ y,
                                                      const float* __restrict__ w, int64_t m, int d, float eps,
                                                      uint32_t* zero, int zero_n) {
  pdl_wait();
  pdl_launch_dependents();
  // words a later kernel needs cleared (its counters), done here so that no
  // memset sits between kernels and breaks their programmatic launches
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < zero_n; i += blockDim.x) zero[i] = 0u;
  constexpr int V = 16 / sizeof(T);
  const int lane = threadIdx.x & 31;
  const int64_t r = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (r >= m) return;  // warp-uniform
  const int nv = d / V;
  const uint4* xr = reinterpret_cast<const uint4*>(x + r * d);
  uint4* yr = reinterpret_cast<uint4*>(y + r * d);
  uint4 v[MAXV];
  float ss = 0.0f;
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int c = lane + 32 * i;
    v[i] = c < nv ? __ldg(xr + c) : make_uint4(0, 0, 0, 0);
  }
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const T* e = reinterpret_cast<const T*>(&v[i]);
#pragma unroll
    for (int t = 0; t < V; ++t) {
      const float f = to_f32(e[t]);
      ss = fmaf(f, f, ss);
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float inv = 1.0f / sqrtf(ss / static_cast<float>(d) + eps);
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int c = lane + 32 * i;
    if (c >= nv) continue;
    float wv[V];
#pragma unroll
    for (int t = 0; t < V; t += 4) {
      const float4 w4 = w ? __ldg(reinterpret_cast<const float4*>(w + c * V + t)) : make_float4(1.0f, 1.0f, 1.0f, 1.0f);
      wv[t] = w4.x;
      wv[t + 1] = w4.y;
      wv[t + 2] = w4.z;
      wv[t + 3] = w4.w;
    }
    const T* e = reinterpret_cast<const T*>(&v[i]);
    uint4 o;
    T* oe = reinterpret_cast<T*>(&o);
#pragma unroll
    for (int t = 0; t < V; ++t) oe[t] = from_f32<T>(to_f32(e[t]) * inv * wv[t]);
    yr[c] = o;
  }
}

// ---------------------------------------------------------------------------
// Per-head q/k RMSNorm (optional) and rotate-half RoPE at the original token
// positions, one warp per row: lane l owns frequencies l*E .. l*E+E-1 of every
// rotated head.  The frequencies theta^(-2i/D) come from the host in double
// precision; the angle pos * f is formed and reduced modulo 2 pi in double
// (positions reach 2^17), so the float sin/cos of the remainder in [-pi, pi]
// is accurate to about 4e-7.
// The hq + hkv heads of the row are processed eight at a time with all their
// loads in flight.
// ---------------------------------------------------------------------------
struct RopeTable {
  double inv_freq[64];  // D / 2 entries
};

template <typename T, int D>
__global__ void __launch_bounds__(256) k_qk_norm_rope_warp(T* __restrict__ qkv, int64_t ld, int m, int hq, int hkv,
                                                           const int32_t* __restrict__ pos,
                                                           const float* __restrict__ wq, const float* __restrict__ wk,
                                                           int qk_norm, float eps,
                                                           const __grid_constant__ RopeTable tab) {
  pdl_wait();
  pdl_launch_dependents();
  constexpr int H2 = D / 2;
  constexpr int E = H2 / 32;
  constexpr int HU = 8;  // heads in flight
  const int lane = threadIdx.x & 31;
  const int r = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (r >= m) return;  // warp-uniform
  const double p = static_cast<double>(pos ? pos[r] : r);
  float cs[E], sn[E], wqa[E], wqb[E], wka[E], wkb[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const double ang = p * tab.inv_freq[lane * E + e];
    const double turns = rint(ang * 0.15915494309189535);  // 1 / (2 pi)
    const float red = static_cast<float>(fma(-turns, 6.283185307179586, ang));
    __sincosf(red, &sn[e], &cs[e]);  // |red| <= pi: absolute error about 4e-7
    wqa[e] = qk_norm ? wq[lane * E + e] : 1.0f;
    wqb[e] = qk_norm ? wq[H2 + lane * E + e] : 1.0f;
    wka[e] = qk_norm ? wk[lane * E + e] : 1.0f;
    wkb[e] = qk_norm ? wk[H2 + lane * E + e] : 1.0f;
  }
  T* row = qkv + static_cast<int64_t>(r) * ld;
  const int heads = hq + hkv;
  for (int h0 = 0; h0 < heads; h0 += HU) {
    float a[HU][E], b[HU][E];
#pragma unroll
    for (int u = 0; u < HU; ++u) {
      const T* x = row + static_cast<int64_t>(h0 + u) * D;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        a[u][e] = h0 + u < heads ? to_f32(x[lane * E + e]) : 0.0f;
        b[u][e] = h0 + u < heads ? to_f32(x[H2 + lane * E + e]) : 0.0f;
      }
    }
#pragma unroll
    for (int u = 0; u < HU; ++u) {
      const int hh = h0 + u;
      if (hh >= heads) break;  // warp-uniform
      const bool isq = hh < hq;
      if (qk_norm) {
        float ss = 0.0f;
#pragma unroll
        for (int e = 0; e < E; ++e) ss += a[u][e] * a[u][e] + b[u][e] * b[u][e];
#pragma unroll
        for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        const float inv = 1.0f / sqrtf(ss / static_cast<float>(D) + eps);
#pragma unroll
        for (int e = 0; e < E; ++e) {
          a[u][e] *= inv * (isq ? wqa[e] : wka[e]);
          b[u][e] *= inv * (isq ? wqb[e] : wkb[e]);
        }
      }
      T* x = row + static_cast<int64_t>(hh) * D;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        x[lane * E + e] = from_f32<T>(a[u][e] * cs[e] - b[u][e] * sn[e]);
        x[H2 + lane * E + e] = from_f32<T>(b[u][e] * cs[e] + a[u][e] * sn[e]);
      }
    }
  }
}

// gu[r][f] <- SiLU(gu[r][f]) * gu[r][d_ff + f]  (rows of 2*d_ff: gate half, then up half)
template <typename T>
__global__ void __launch_bounds__(256) k_swiglu(T* __restrict__ gu, int64_t m, int d_ff) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
  if (i >= m * d_ff) return;
  const int64_t r = i / d_ff;
  const int f = static_cast<int>(i - r * d_ff);
  T* row = gu + r * 2 * d_ff;
  const float g = to_f32(row[f]);
  const float u = to_f32(row[d_ff + f]);
  row[f] = from_f32<T>(g / (1.0f + expf(-g)) * u);
}

}  // namespace tg

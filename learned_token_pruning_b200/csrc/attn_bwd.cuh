// Backward of token-gated causal GQA attention ("TokenGate and T2Quant: a
// close reading", §4.1 engineering notes: the biased attention kernel also
// accumulates the bias gradient back into the scorer).  With
//     l_rc = a_r z_rc + gain_h bias_c,  a_r = temp_h ratio_r,  z_rc = sm_scale q_r . k_c   (c <= r)
//     P = softmax_c(l),  o_r = sum_c P_rc v_c,  dO given:
//     dP_rc = dO_r . v_c,   dl_rc = P_rc (dP_rc - dO_r . o_r)
//     dq_r = sum_c dl_rc a_r sm_scale k_c          dk_c = sum_{h in group, r} dl_rc a_r sm_scale q_r
//     dv_c = sum_{h in group, r} P_rc dO_r         dbias_c = sum_h gain_h sum_r dl_rc
//     dgain_h = sum_{r,c} dl_rc bias_c             dtemp_h = sum_{r,c} dl_rc ratio_r z_rc
// P is recomputed from the forward's log-sum-exp.  CUDA cores, fp32, and
// deterministic: every gradient element is written by one thread of one CTA,
// and the cross-CTA sums (dbias over KV heads, dgain / dtemp over key blocks)
// go through the workspace and are added in a fixed order.
//   k_attn_bwd_rowdot   D_hr = dO_r . o_r per head and row (one warp each)
//   k_attn_bwd_kv       CTA (g, key block of 32): dk, dv of the block for KV
//                       head g, walking the query tiles of 32 rows at or
//                       after the block for each head of g's group; partial
//                       dbias (per key, over the group's heads) and partial
//                       dgain / dtemp (per head, over the block's keys)
//   k_attn_bwd_q        CTA (h, query block of 32): dq, walking the key
//                       blocks up to the diagonal
//   k_attn_bwd_final    the fixed-order sums of the partials
#pragma once

#include "common.cuh"
#include "simt.cuh"

namespace tg {

constexpr int kBwdBlk = 32;       // rows of a query tile = keys of a key block
constexpr int kBwdThreads = 256;  // thread t: tile row / key t / 8, a quarter of the other operand

struct AttnBwdParams {
  const void *q, *k, *v, *o, *dout;
  int64_t ldq, ldk, ldv, ldo, lddo;
  int m, hq, hkv, group;
  const float* bias;   // [m] or null
  const float* gain;   // [hq]
  const float* temp;   // [hq]
  const float* ratio;  // [m] or null
  const float* lse;    // [hq][m], natural log
  float sm_scale;
  float* dq;           // [m][hq*D]
  float* dk;           // [m][hkv*D]
  float* dv;           // [m][hkv*D]
  float* dbias;        // [m] or null
  float* dgain;        // [hq] or null
  float* dtemp;        // [hq] or null
  float* rowdot;       // workspace [hq][m]
  float* dbias_part;   // workspace [hkv][m]
  float* dgt_part;     // workspace [hq][nkb][2]: (dgain, dtemp) partials
  int nkb;             // key blocks
  float* rowpar;       // workspace [hq][m_pad / 2][8] (tensor-core kernels): per-row constants of row pairs
  int m_pad;           // m rounded up to 128
  int dbias_nparts;    // rows of dbias_part summed into dbias (hkv here, hq for the tensor-core kernels)
  float* kv_part;      // workspace [hkv * m_pad / 128][group][128][2 D]: one head's (dV, dK) of a key block
  unsigned* kv_ctr;    // workspace [2][hkv * m_pad / 128]: tickets, partials published; zero on entry
};

template <typename T>
__device__ __forceinline__ float ld_f32(const void* base, int64_t idx) {
  return to_f32(static_cast<const T*>(base)[idx]);
}

template <typename T, int D>
__global__ void __launch_bounds__(256) k_attn_bwd_rowdot(AttnBwdParams p) {
  const int w = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (w >= p.m * p.hq) return;  // warp-uniform
  const int r = w / p.hq, h = w % p.hq;
  float s = 0.0f;
  for (int d = lane; d < D; d += 32)
    s = fmaf(ld_f32<T>(p.dout, int64_t(r) * p.lddo + h * D + d), ld_f32<T>(p.o, int64_t(r) * p.ldo + h * D + d), s);
#pragma unroll
  for (int off = 16; off; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if (lane == 0) p.rowdot[int64_t(h) * p.m + r] = s;
}

// Scores of a 32 x 32 tile: thread t takes row t / 8 and keys 4 (t % 8) .. + 3.
// Returns P and dl of those four entries (0 where masked or out of range).
template <int D, int DP>
__device__ __forceinline__ void bwd_tile_scores(const AttnBwdParams& p, const float* Qs, const float* dOs,
                                                const float* Ks, const float* Vs, int h, int row0, int key0,
                                                float (&pr)[4], float (&dl)[4], float (&zz)[4]) {
  const int t = threadIdx.x, r = t >> 3, c0 = (t & 7) * 4;
  const int gr = row0 + r;
  float s[4] = {0, 0, 0, 0}, dp[4] = {0, 0, 0, 0};
  for (int d = 0; d < D; ++d) {
    const float qv = Qs[r * DP + d], gv = dOs[r * DP + d];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      s[j] = fmaf(qv, Ks[(c0 + j) * DP + d], s[j]);
      dp[j] = fmaf(gv, Vs[(c0 + j) * DP + d], dp[j]);
    }
  }
  const bool row_ok = gr < p.m;
  const float a = row_ok ? p.temp[h] * (p.ratio ? p.ratio[gr] : 1.0f) : 0.0f;
  const float lse = row_ok ? p.lse[int64_t(h) * p.m + gr] : 0.0f;
  const float D_r = row_ok ? p.rowdot[int64_t(h) * p.m + gr] : 0.0f;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int gc = key0 + c0 + j;
    const bool ok = row_ok && gc < p.m && gc <= gr;
    const float z = s[j] * p.sm_scale;
    const float l = a * z + p.gain[h] * (p.bias && gc < p.m ? p.bias[gc] : 0.0f);
    pr[j] = ok ? __expf(l - lse) : 0.0f;
    dl[j] = ok ? pr[j] * (dp[j] - D_r) : 0.0f;
    zz[j] = ok ? z : 0.0f;
  }
}

// Stage rows [row0, row0 + 32) of head column col0 of a [m][ld] tensor into s (stride DP), zero past m.
template <typename T, int D, int DP>
__device__ __forceinline__ void bwd_stage(float* s, const void* src, int64_t ld, int col0, int row0, int m) {
  for (int i = threadIdx.x; i < kBwdBlk * D; i += kBwdThreads) {
    const int r = i / D, d = i % D;
    s[r * DP + d] = row0 + r < m ? ld_f32<T>(src, int64_t(row0 + r) * ld + col0 + d) : 0.0f;
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(kBwdThreads) k_attn_bwd_kv(AttnBwdParams p) {
  constexpr int DP = D + 1;
  extern __shared__ float bwd_smem[];
  float* Ks = bwd_smem;
  float* Vs = Ks + kBwdBlk * DP;
  float* Qs = Vs + kBwdBlk * DP;
  float* dOs = Qs + kBwdBlk * DP;
  float* Ps = dOs + kBwdBlk * DP;              // [32 rows][33]
  float* dSs = Ps + kBwdBlk * (kBwdBlk + 1);   // [32 rows][33], dl * a_r * sm_scale
  float* dLs = dSs + kBwdBlk * (kBwdBlk + 1);  // [32 rows][33], dl
  float* red = dLs + kBwdBlk * (kBwdBlk + 1);  // [256] reduction scratch
  const int g = blockIdx.x / p.nkb, kb = blockIdx.x % p.nkb;
  const int key0 = kb * kBwdBlk;
  const int t = threadIdx.x;
  bwd_stage<T, D, DP>(Ks, p.k, p.ldk, g * D, key0, p.m);
  bwd_stage<T, D, DP>(Vs, p.v, p.ldv, g * D, key0, p.m);
  // thread t accumulates dk / dv of key t / 8, dims (t % 8) * (D / 8) ..
  constexpr int DC = D / 8;
  const int kc = t >> 3, d0 = (t & 7) * DC;
  float dk[DC], dv[DC];
#pragma unroll
  for (int i = 0; i < DC; ++i) dk[i] = dv[i] = 0.0f;
  float dbias_acc = 0.0f;  // for key t (t < 32), summed over the group's heads
  for (int u = 0; u < p.group; ++u) {
    const int h = g * p.group + u;
    float dgain_acc = 0.0f, dtemp_acc = 0.0f;
    for (int row0 = key0; row0 < p.m; row0 += kBwdBlk) {
      __syncthreads();  // the previous tile's smem is consumed
      bwd_stage<T, D, DP>(Qs, p.q, p.ldq, h * D, row0, p.m);
      bwd_stage<T, D, DP>(dOs, p.dout, p.lddo, h * D, row0, p.m);
      __syncthreads();
      float pr[4], dl[4], zz[4];
      bwd_tile_scores<D, DP>(p, Qs, dOs, Ks, Vs, h, row0, key0, pr, dl, zz);
      const int r = t >> 3, c0 = (t & 7) * 4, gr = row0 + r;
      const float as = gr < p.m ? p.temp[h] * (p.ratio ? p.ratio[gr] : 1.0f) * p.sm_scale : 0.0f;
      const float rr = gr < p.m ? (p.ratio ? p.ratio[gr] : 1.0f) : 0.0f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        Ps[r * (kBwdBlk + 1) + c0 + j] = pr[j];
        dSs[r * (kBwdBlk + 1) + c0 + j] = dl[j] * as;
        dLs[r * (kBwdBlk + 1) + c0 + j] = dl[j];
        const int gc = key0 + c0 + j;
        dgain_acc = fmaf(dl[j], p.bias && gc < p.m ? p.bias[gc] : 0.0f, dgain_acc);
        dtemp_acc = fmaf(dl[j], rr * zz[j], dtemp_acc);
      }
      __syncthreads();
      // dv[c][d] += sum_r P[r][c] dO[r][d];  dk[c][d] += sum_r dS[r][c] q[r][d]
      for (int rr2 = 0; rr2 < kBwdBlk; ++rr2) {
        const float pv = Ps[rr2 * (kBwdBlk + 1) + kc], sv = dSs[rr2 * (kBwdBlk + 1) + kc];
#pragma unroll
        for (int i = 0; i < DC; ++i) {
          dv[i] = fmaf(pv, dOs[rr2 * DP + d0 + i], dv[i]);
          dk[i] = fmaf(sv, Qs[rr2 * DP + d0 + i], dk[i]);
        }
      }
      if (t < kBwdBlk) {
        float sacc = 0.0f;
        for (int rr2 = 0; rr2 < kBwdBlk; ++rr2) sacc += dLs[rr2 * (kBwdBlk + 1) + t];
        dbias_acc = fmaf(p.gain[h], sacc, dbias_acc);
      }
    }
    // per-head partials of dgain / dtemp over this key block (fixed-order block reduction)
    __syncthreads();
    red[t] = dgain_acc;
    __syncthreads();
    for (int s2 = kBwdThreads / 2; s2; s2 >>= 1) {
      if (t < s2) red[t] += red[t + s2];
      __syncthreads();
    }
    if (t == 0) p.dgt_part[(int64_t(h) * p.nkb + kb) * 2] = red[0];
    __syncthreads();
    red[t] = dtemp_acc;
    __syncthreads();
    for (int s2 = kBwdThreads / 2; s2; s2 >>= 1) {
      if (t < s2) red[t] += red[t + s2];
      __syncthreads();
    }
    if (t == 0) p.dgt_part[(int64_t(h) * p.nkb + kb) * 2 + 1] = red[0];
  }
  const int gc = key0 + kc;
  if (gc < p.m) {
#pragma unroll
    for (int i = 0; i < DC; ++i) {
      p.dk[int64_t(gc) * p.hkv * D + g * D + d0 + i] = dk[i];
      p.dv[int64_t(gc) * p.hkv * D + g * D + d0 + i] = dv[i];
    }
  }
  if (t < kBwdBlk && key0 + t < p.m) p.dbias_part[int64_t(g) * p.m + key0 + t] = dbias_acc;
}

template <typename T, int D>
__global__ void __launch_bounds__(kBwdThreads) k_attn_bwd_q(AttnBwdParams p) {
  constexpr int DP = D + 1;
  extern __shared__ float bwd_smem[];
  float* Ks = bwd_smem;
  float* Vs = Ks + kBwdBlk * DP;
  float* Qs = Vs + kBwdBlk * DP;
  float* dOs = Qs + kBwdBlk * DP;
  float* dSs = dOs + kBwdBlk * DP;  // [32 rows][33], dl * a_r * sm_scale
  const int nqb = (p.m + kBwdBlk - 1) / kBwdBlk;
  const int h = blockIdx.x / nqb, qb = blockIdx.x % nqb;
  const int g = h / p.group;
  const int row0 = qb * kBwdBlk;
  const int t = threadIdx.x;
  bwd_stage<T, D, DP>(Qs, p.q, p.ldq, h * D, row0, p.m);
  bwd_stage<T, D, DP>(dOs, p.dout, p.lddo, h * D, row0, p.m);
  constexpr int DC = D / 8;
  const int qr = t >> 3, d0 = (t & 7) * DC;
  float dq[DC];
#pragma unroll
  for (int i = 0; i < DC; ++i) dq[i] = 0.0f;
  for (int key0 = 0; key0 <= row0 && key0 < p.m; key0 += kBwdBlk) {
    __syncthreads();
    bwd_stage<T, D, DP>(Ks, p.k, p.ldk, g * D, key0, p.m);
    bwd_stage<T, D, DP>(Vs, p.v, p.ldv, g * D, key0, p.m);
    __syncthreads();
    float pr[4], dl[4], zz[4];
    bwd_tile_scores<D, DP>(p, Qs, dOs, Ks, Vs, h, row0, key0, pr, dl, zz);
    const int r = t >> 3, c0 = (t & 7) * 4, gr = row0 + r;
    const float as = gr < p.m ? p.temp[h] * (p.ratio ? p.ratio[gr] : 1.0f) * p.sm_scale : 0.0f;
#pragma unroll
    for (int j = 0; j < 4; ++j) dSs[r * (kBwdBlk + 1) + c0 + j] = dl[j] * as;
    __syncthreads();
    // dq[r][d] += sum_c dS[r][c] k[c][d]
    for (int c = 0; c < kBwdBlk; ++c) {
      const float sv = dSs[qr * (kBwdBlk + 1) + c];
#pragma unroll
      for (int i = 0; i < DC; ++i) dq[i] = fmaf(sv, Ks[c * DP + d0 + i], dq[i]);
    }
  }
  const int gr = row0 + qr;
  if (gr < p.m) {
#pragma unroll
    for (int i = 0; i < DC; ++i) p.dq[int64_t(gr) * p.hq * D + h * D + d0 + i] = dq[i];
  }
}

__global__ void __launch_bounds__(256) k_attn_bwd_final(AttnBwdParams p) {
  const int i = blockIdx.x * 256 + threadIdx.x;
  if (p.dbias && i < p.m) {
    float s = 0.0f;
    for (int g = 0; g < p.dbias_nparts; ++g) s += p.dbias_part[int64_t(g) * p.m + i];
    p.dbias[i] = s;
  }
  if (i < p.hq) {
    float sg = 0.0f, st = 0.0f;
    for (int kb = 0; kb < p.nkb; ++kb) {
      sg += p.dgt_part[(int64_t(i) * p.nkb + kb) * 2];
      st += p.dgt_part[(int64_t(i) * p.nkb + kb) * 2 + 1];
    }
    if (p.dgain) p.dgain[i] = sg;
    if (p.dtemp) p.dtemp[i] = st;
  }
}

}  // namespace tg

// Compaction of the kept rows and the per-row inputs of token-gated attention.
//
// "TokenGate and T2Quant: a close reading", §4.1: the layers above the gate
// process only the kept tokens; the importance b_j = s_j / rms_seq(s) becomes
// the key bias of token-gated attention, and the temperature factor of kept row
// i is log m_i / log max(2, p_i) with m_i = i + 1 (rank among kept tokens) and
// p_i = idx_i + 1 (original position).
//
// k_gather_bulk moves whole rows with the bulk-copy (TMA) engine: one thread
// per CTA streams batches of rows global -> shared -> global through two
// shared-memory halves (loads of batch b+1 overlap the stores of batch b)
// while the other threads write the per-row side outputs.  k_gather (16-byte
// vector copies by every thread) handles rows too large for the staging buffer.
#pragma once

#include "common.cuh"

namespace tg {

constexpr int kGatherThreads = 256;
constexpr int kGatherRows = 4;
constexpr int kGatherUnroll = 4;

struct GatherParams {
  const uint8_t* hidden;
  int64_t n;
  int64_t row_bytes;  // multiple of 16
  const int32_t* idx;
  int64_t m;
  const float* scores;
  const float* sumsq;
  int64_t n_prunable;
  float eps;
  uint8_t* out;
  int32_t* pos;
  float* bias;
  float* ratio;
  uint32_t* zero;  // k_gather_rmsnorm_warp: words cleared by block 0 for a later kernel (or null)
  int zero_n;
};

__global__ void __launch_bounds__(kGatherThreads) k_gather(GatherParams p) {
  pdl_wait();
  pdl_launch_dependents();
  __shared__ int64_t src_row[kGatherRows];
  const int64_t r0 = static_cast<int64_t>(blockIdx.x) * kGatherRows;
  const int tid = threadIdx.x;
  if (tid < kGatherRows) {
    const int64_t r = r0 + tid;
    int64_t j = -1;
    if (r < p.m) {
      j = p.idx[r];
      if (j < 0 || j >= p.n) {
        raise_error(kErrGatherIndex, static_cast<uint32_t>(r & 0xffffff));
        j = -1;
      } else {
        if (p.pos) p.pos[r] = static_cast<int32_t>(j);
        if (p.bias) {
          const float rms = sqrtf(p.sumsq[0] / static_cast<float>(p.n_prunable) + p.eps);
          p.bias[r] = p.scores[j] / rms;
        }
        if (p.ratio) {
          const double lm = log(static_cast<double>(r + 1));
          const double lp = log(fmax(2.0, static_cast<double>(j) + 1.0));
          p.ratio[r] = static_cast<float>(lm / lp);
        }
      }
    }
    src_row[tid] = j;
  }
  __syncthreads();

  const int64_t units = p.row_bytes / 16;
  const int64_t rows_here = min(static_cast<int64_t>(kGatherRows), p.m - r0);
  const int64_t total = rows_here * units;
  for (int64_t base = 0; base < total; base += static_cast<int64_t>(kGatherThreads) * kGatherUnroll) {
    uint4 v[kGatherUnroll];
    int64_t dst[kGatherUnroll];
#pragma unroll
    for (int u = 0; u < kGatherUnroll; ++u) {
      const int64_t e = base + tid + static_cast<int64_t>(u) * kGatherThreads;
      dst[u] = -1;
      if (e < total) {
        const int64_t rr = e / units, cu = e - rr * units;
        const int64_t j = src_row[rr];
        if (j >= 0) {
          v[u] = __ldg(reinterpret_cast<const uint4*>(p.hidden + j * p.row_bytes) + cu);
          dst[u] = (r0 + rr) * p.row_bytes + cu * 16;
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kGatherUnroll; ++u) {
      if (dst[u] >= 0) *reinterpret_cast<uint4*>(p.out + dst[u]) = v[u];
    }
  }
}

constexpr int kGatherBulkThreads = 128;
constexpr int kGatherBatch = 8;                    // rows per bulk batch
constexpr size_t kGatherStageBytes = 96 * 1024;    // both halves of the staging buffer

__device__ __forceinline__ void gather_side_outputs(const GatherParams& p, int64_t r, int64_t j) {
  if (p.pos) p.pos[r] = static_cast<int32_t>(j);
  if (p.bias) {
    const float rms = sqrtf(p.sumsq[0] / static_cast<float>(p.n_prunable) + p.eps);
    p.bias[r] = p.scores[j] / rms;
  }
  if (p.ratio) {
    const double lm = log(static_cast<double>(r + 1));
    const double lp = log(fmax(2.0, static_cast<double>(j) + 1.0));
    p.ratio[r] = static_cast<float>(lm / lp);
  }
}

// rows_per_batch * row_bytes * 2 <= dynamic shared memory; rows [r_begin, r_end) per CTA.
__global__ void __launch_bounds__(kGatherBulkThreads) k_gather_bulk(GatherParams p, int rows_per_batch) {
  pdl_wait();
  pdl_launch_dependents();
  extern __shared__ __align__(128) uint8_t gbuf[];
  __shared__ uint64_t bar[2];
  const int64_t per = (p.m + gridDim.x - 1) / gridDim.x;
  const int64_t r_begin = static_cast<int64_t>(blockIdx.x) * per;
  const int64_t r_end = min(p.m, r_begin + per);
  if (threadIdx.x == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    fence_mbar_init();
  }
  __syncthreads();
  // per-row side outputs (every thread but the copy issuer)
  for (int64_t r = r_begin + threadIdx.x - 1; threadIdx.x > 0 && r < r_end; r += kGatherBulkThreads - 1) {
    const int64_t j = p.idx[r];
    if (j < 0 || j >= p.n) {
      raise_error(kErrGatherIndex, static_cast<uint32_t>(r & 0xffffff));
      continue;
    }
    gather_side_outputs(p, r, j);
  }
  if (threadIdx.x != 0) return;
  // the copy issuer
  const uint32_t rb = static_cast<uint32_t>(p.row_bytes);
  int batch = 0;
  bool ok = true;
  for (int64_t r0 = r_begin; r0 < r_end && ok; r0 += rows_per_batch, ++batch) {
    const int b = batch & 1;
    const int cnt = static_cast<int>(min(static_cast<int64_t>(rows_per_batch), r_end - r0));
    uint8_t* half = gbuf + static_cast<size_t>(b) * rows_per_batch * rb;
    // this half was last read by the stores of batch - 2: keep at most the
    // newest group (batch - 1) in flight
    bulk_wait_read<1>();
    int64_t src[kGatherBatch];
    uint32_t bytes = 0;
    for (int i = 0; i < cnt; ++i) {
      const int64_t j = p.idx[r0 + i];
      src[i] = (j >= 0 && j < p.n) ? j : -1;  // a bad index was reported above; its row is skipped
      if (src[i] >= 0) bytes += rb;
    }
    mbar_arrive_expect_tx(&bar[b], bytes);
    for (int i = 0; i < cnt; ++i)
      if (src[i] >= 0) bulk_load(half + static_cast<size_t>(i) * rb, p.hidden + src[i] * p.row_bytes, rb, &bar[b]);
    ok = mbar_wait(&bar[b], (batch >> 1) & 1, kErrWaitGather);
    if (!ok) break;
    for (int i = 0; i < cnt; ++i)
      if (src[i] >= 0) bulk_store(p.out + (r0 + i) * p.row_bytes, half + static_cast<size_t>(i) * rb, rb);
    bulk_commit();
  }
  bulk_wait_all();
}

}  // namespace tg

namespace tg {

// ---------------------------------------------------------------------------
// Gather fused with the first RMSNorm of the layer that reads the kept rows.
// One warp per kept row r: the source row hidden[idx[r]] is loaded once into
// registers (every 16-byte load of a lane in flight together), written out
// unchanged as the residual copy hidden_kept[r] (bit-exact, as k_gather_bulk),
// and normalised in the same pass, xn[r] = x / sqrt(mean(x^2) + eps) * w,
// rounded to the row's dtype (the arithmetic and summation order of
// k_rmsnorm_warp, so the result equals a gather followed by that norm).
// Lane 0 writes the side outputs pos, bias and ratio as k_gather_bulk does.
// ---------------------------------------------------------------------------
template <typename T, int MAXV>
__global__ void __launch_bounds__(256) k_gather_rmsnorm_warp(GatherParams p, T* __restrict__ xn,
                                                             const float* __restrict__ w, int d, float norm_eps) {
  pdl_wait();
  pdl_launch_dependents();
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < p.zero_n; i += blockDim.x) p.zero[i] = 0u;
  constexpr int V = 16 / sizeof(T);
  const int lane = threadIdx.x & 31;
  const int64_t r = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (r >= p.m) return;  // warp-uniform
  const int64_t j = p.idx[r];
  if (j < 0 || j >= p.n) {
    if (lane == 0) raise_error(kErrGatherIndex, static_cast<uint32_t>(r & 0xffffff));
    return;
  }
  const int nv = d / V;
  const uint4* xr = reinterpret_cast<const uint4*>(p.hidden + j * p.row_bytes);
  uint4* cr = reinterpret_cast<uint4*>(p.out + r * p.row_bytes);
  uint4* yr = reinterpret_cast<uint4*>(xn + r * d);
  uint4 v[MAXV];
  float ss = 0.0f;
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int c = lane + 32 * i;
    v[i] = c < nv ? __ldg(xr + c) : make_uint4(0, 0, 0, 0);
  }
  if (lane == 0) gather_side_outputs(p, r, j);
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int c = lane + 32 * i;
    if (c < nv) cr[c] = v[i];
    const T* e = reinterpret_cast<const T*>(&v[i]);
#pragma unroll
    for (int t = 0; t < V; ++t) {
      const float f = to_f32(e[t]);
      ss = fmaf(f, f, ss);
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float inv = 1.0f / sqrtf(ss / static_cast<float>(d) + norm_eps);
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

}  // namespace tg

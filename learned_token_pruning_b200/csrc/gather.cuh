// Compaction of the kept rows and the per-row inputs of token-gated attention.
//
// "TokenGate and T2Quant: a close reading", §4.1: the layers above the gate
// process only the kept tokens; the importance b_j = s_j / rms_seq(s) becomes
// the key bias of token-gated attention, and the temperature factor of kept row
// i is log m_i / log max(2, p_i) with m_i = i + 1 (rank among kept tokens) and
// p_i = idx_i + 1 (original position).
//
// Each CTA copies kGatherRows rows with 16-byte vector loads, all loads of a
// thread issued before its stores so several are in flight per thread.
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
};

__global__ void __launch_bounds__(kGatherThreads) k_gather(GatherParams p) {
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

}  // namespace tg

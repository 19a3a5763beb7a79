// Masked top-K selection with stable compaction.
//
// TokenGate keeps S = top-K(b_j) over the prunable (document) tokens plus
// every non-prunable (question) token ("TokenGate and T2Quant: a close
// reading", §4.1 "Top-K selector").  The kept set must come out identical to a
// full stable sort by (score desc, index asc), so the selection runs on
// integer keys that order fp32 scores totally:
//   -0 and +0 map to the same key, NaN maps below -inf, larger score = larger key.
//
// Longer prompts take one thread-block cluster of up to kSelCluster CTAs, each
// owning a contiguous slice of the tokens with its keys cached in shared
// memory.  The threshold key T (the kp-th largest prunable key) is found in
// two steps:
//   1. its top 11 bits d1, from a histogram of (key >> 21) over the prunable
//      tokens: the gate-score kernel's, or one the CTAs build and merge
//      through distributed shared memory;
//   2. its low 21 bits, among the candidates (the keys whose top 11 bits are
//      d1, usually a few percent of the tokens): every CTA gathers all
//      candidates into its own shared memory and finds the bits with three
//      7-bit radix passes that need only block-level barriers.
// Should the candidates not fit, the low bits take three cluster-wide radix
// passes instead.  Each CTA then counts its tokens kept outright (key > T, or
// non-prunable) and its ties at T, pushes both counts into every CTA's shared
// memory, and after one cluster barrier writes its kept indices in ascending
// order (ties at T towards the lower index), thread t owning the consecutive
// tokens [t*kpt, (t+1)*kpt) of the slice so that one block scan places them.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"

namespace tg {

namespace cg = cooperative_groups;

constexpr int kSelCluster = 16;  // 16 needs the non-portable cluster size (the host falls back to 8)
constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kSelStride = kSelThreads + 1;  // words per row of the key cache [kpt][kSelStride]
constexpr int kSelMaxKpt = 32;               // cached slices hold up to kSelMaxKpt tokens per thread
constexpr int kSelOwnCap = 8192;             // candidate keys one CTA can publish
constexpr int kSelAllCap = 16384;            // candidate keys one CTA can gather
constexpr size_t kSelCandBytes = static_cast<size_t>(kSelOwnCap + kSelAllCap) * 4;
constexpr int kSelTopBits = 11;              // first digit: key bits 31..21
constexpr int kSelLowBits = 7;               // the other 21 bits: three digits of 7

struct SelectParams {
  const float* scores;
  const uint8_t* prunable;
  int64_t n;
  int64_t n_prunable;
  int64_t k;
  int32_t* out;
  int64_t m;
  int64_t slice;  // tokens per CTA
  int kpt;        // tokens per thread: a power of two with kpt * kSelThreads >= slice
  int cached;     // 1 if the slice's keys and flags are kept in shared memory (kpt <= kSelMaxKpt)
  const uint32_t* hist_top;  // [2048] counts of (key >> 21) over prunable tokens, or null
  uint32_t* hist_clear;      // hist_top again when it is to be left zeroed for the next call, or null
};

// dynamic shared memory of k_topk_select
__host__ __device__ constexpr size_t select_smem_bytes(int kpt, int cached) {
  return kSelCandBytes + (cached ? ((static_cast<size_t>(kpt) * kSelStride * 5 + 15) / 16) * 16 : 0);
}

// Exclusive scan over the block of one 32-bit value per thread; returns the
// exclusive prefix and writes the block total to *total.
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t* warp_sums, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = lane < kSelWarps ? warp_sums[lane] : 0u;
    uint32_t wx = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t y = __shfl_up_sync(0xffffffffu, wx, o);
      if (lane >= o) wx += y;
    }
    if (lane < kSelWarps) warp_sums[lane] = wx - w;  // exclusive warp offsets
    if (lane == kSelWarps - 1) warp_sums[kSelWarps] = wx;
  }
  __syncthreads();
  const uint32_t r = warp_sums[warp] + x - v;
  *total = warp_sums[kSelWarps];
  __syncthreads();
  return r;
}

// One warp over 128 bins, lane l holding the counts of bins 127-4l .. 124-4l
// (highest first) in v[0..3]: the bin holding the rem-th largest key and the
// count of keys in the bins above it go to s_pick[0], s_pick[1].  Lane 0 sets
// s_pick to (0, 0) first, so counts that cannot hold rem leave an in-range digit.
__device__ __forceinline__ void warp_pick_low_digit(const uint32_t v[4], uint32_t rem, uint32_t* s_pick) {
  const int lane = threadIdx.x & 31;
  if (lane == 0) {
    s_pick[0] = 0;
    s_pick[1] = 0;
  }
  __syncwarp();
  const uint32_t c = v[0] + v[1] + v[2] + v[3];
  uint32_t incl = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const uint32_t above = incl - c;
  if (above < rem && rem <= incl) {
    uint32_t a = above;
    int u = 0;
    for (; u < 3 && a + v[u] < rem; ++u) a += v[u];
    s_pick[0] = static_cast<uint32_t>(127 - 4 * lane - u);
    s_pick[1] = a;
  }
}

__global__ void __launch_bounds__(kSelThreads, 1) k_topk_select(SelectParams p) {
  pdl_wait();
  pdl_launch_dependents();
  extern __shared__ __align__(16) uint8_t sel_smem[];
  __shared__ __align__(16) uint32_t hist[1 << kSelTopBits];  // this CTA's first-digit counts
  __shared__ uint32_t lhist[3][1 << kSelLowBits];  // the candidates' counts, one array per low digit
  __shared__ uint32_t warp_sums[kSelWarps + 1];
  __shared__ uint32_t info_a[kSelCluster][2];  // written by rank r into every rank: its prunable count, its candidates
  __shared__ uint32_t info_b[kSelCluster][2];  // written by rank r into every rank: tokens it keeps outright, its ties at T
  __shared__ uint32_t s_pick[2];
  __shared__ uint32_t s_ncand;
  __shared__ uint32_t s_off[kSelCluster];
  __shared__ uint32_t s_lpick[3][2];

  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int nranks = static_cast<int>(cluster.num_blocks());
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t lo = static_cast<int64_t>(rank) * p.slice;
  const int64_t hi = min(p.n, lo + p.slice);
  const int64_t len = hi > lo ? hi - lo : 0;
  const int kpt = p.kpt;
  const int kshift = __ffs(kpt) - 1;
  const bool top = p.hist_top != nullptr;

  uint32_t* own_cand = reinterpret_cast<uint32_t*>(sel_smem);  // [kSelOwnCap] read by every rank
  uint32_t* all_cand = own_cand + kSelOwnCap;                   // [kSelAllCap]
  uint32_t* keys = all_cand + kSelAllCap;                       // [kpt][kSelStride]: token t*kpt + j at j*kSelStride + t
  uint8_t* flags = reinterpret_cast<uint8_t*>(keys + static_cast<size_t>(kpt) * kSelStride);

  // token i = tid*kpt + j of the slice (the caller checks i < len)
  auto load_own = [&](int j, uint32_t& key, bool& f) {
    if (p.cached) {
      const int s = j * kSelStride + tid;
      key = keys[s];
      f = flags[s] != 0;
    } else {
      const int64_t g = lo + static_cast<int64_t>(tid) * kpt + j;
      f = p.prunable[g] != 0;
      key = f ? order_key(p.scores[g]) : 0u;
    }
  };

  if (tid == 0) {
    s_ncand = 0;
    s_pick[0] = 0;
    s_pick[1] = 0;
  }
  if (tid < 3 * (1 << kSelLowBits)) (&lhist[0][0])[tid] = 0;
  if (tid < 6) (&s_lpick[0][0])[tid] = 0;
  // the first-digit counts, four bins a thread with the highest first: thread
  // t holds bins 2047-4t .. 2044-4t
  uint32_t hv[4] = {0u, 0u, 0u, 0u};
  if (top) {
    const uint4 q = __ldg(reinterpret_cast<const uint4*>(p.hist_top) + (kSelThreads - 1 - tid));
    hv[0] = q.w;
    hv[1] = q.z;
    hv[2] = q.y;
    hv[3] = q.x;
  } else {
    for (int b = tid; b < (1 << kSelTopBits); b += kSelThreads) hist[b] = 0;
  }
  // the first round of the slice's loads goes out before anything waits
  float sc[4];
  uint8_t pf[4];
  auto issue = [&](int64_t base) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t i = base + u * kSelThreads + tid;
      sc[u] = i < len ? __ldg(p.scores + lo + i) : 0.0f;
      pf[u] = i < len ? __ldg(p.prunable + lo + i) : uint8_t(0);
    }
  };
  issue(0);
  __syncthreads();

  // ---- the first digit from the counts: kp = min(k, prunable tokens), the
  // counts summing to the latter; mode 0: keep no prunable token, 1: keep all
  // of them, 2: threshold select
  uint32_t np_total = 0, kp = 0, d1 = 0, rem = 0;
  int mode = 0;
  auto first_digit = [&]() {
    const uint32_t c4 = hv[0] + hv[1] + hv[2] + hv[3];
    const uint32_t above4 = block_exclusive_scan(c4, warp_sums, &np_total);
    kp = static_cast<uint32_t>(min(p.k, static_cast<int64_t>(np_total)));
    mode = kp == 0 ? 0 : (kp >= np_total ? 1 : 2);
    if (mode == 2 && above4 < kp && kp <= above4 + c4) {
      uint32_t a = above4;
      int u = 0;
      for (; u < 3 && a + hv[u] < kp; ++u) a += hv[u];
      s_pick[0] = static_cast<uint32_t>((1 << kSelTopBits) - 1 - 4 * tid - u);
      s_pick[1] = a;
    }
    __syncthreads();
    d1 = s_pick[0];
    rem = mode == 2 ? kp - s_pick[1] : 0u;  // rank of T among the keys whose first digit is d1
  };
  // warp-aggregated append of this lane's key to the CTA's candidate list
  auto append = [&](bool c, uint32_t key) {
    const uint32_t bal = __ballot_sync(0xffffffffu, c);
    if (bal) {
      const int leader = __ffs(bal) - 1;
      uint32_t b0 = 0;
      if (lane == leader) b0 = atomicAdd(&s_ncand, static_cast<uint32_t>(__popc(bal)));
      b0 = __shfl_sync(0xffffffffu, b0, leader);
      const uint32_t pos = b0 + static_cast<uint32_t>(__popc(bal & ((1u << lane) - 1u)));
      if (c && pos < static_cast<uint32_t>(kSelOwnCap)) own_cand[pos] = key;
    }
  };
  if (top) first_digit();

  // ---- load the slice (coalesced, the next round in flight while one is
  // processed): keys and flags into the cache, the prunable count, and either
  // the candidates (first digit known) or this CTA's first-digit counts
  uint32_t cnt = 0;
  for (int64_t base = 0; base < len; base += 4 * kSelThreads) {
    float csc[4];
    uint8_t cpf[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      csc[u] = sc[u];
      cpf[u] = pf[u];
    }
    if (base + 4 * kSelThreads < len) issue(base + 4 * kSelThreads);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t i = base + u * kSelThreads + tid;
      const bool f = cpf[u] != 0;
      const uint32_t key = f ? order_key(csc[u]) : 0u;
      if (p.cached && i < len) {
        const int s = static_cast<int>(i & (kpt - 1)) * kSelStride + static_cast<int>(i >> kshift);
        keys[s] = key;
        flags[s] = f ? 1 : 0;
      }
      cnt += f ? 1u : 0u;
      if (top) {
        if (mode == 2) append(f && (key >> (32 - kSelTopBits)) == d1, key);
      } else {
        // lanes holding the same digit add once (scores crowd into a few bins)
        const uint32_t bin = f ? (key >> (32 - kSelTopBits)) : 0xffffffffu;
        const uint32_t peers = __match_any_sync(0xffffffffu, bin);
        if (f && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], static_cast<uint32_t>(__popc(peers)));
      }
    }
  }
  uint32_t np_cta;
  block_exclusive_scan(cnt, warp_sums, &np_cta);

  if (!top) {
    cluster.sync();  // every CTA's first-digit counts are complete
    uint4 q[kSelCluster];
#pragma unroll
    for (int r = 0; r < kSelCluster; ++r)
      if (r < nranks) q[r] = reinterpret_cast<const uint4*>(cluster.map_shared_rank(hist, r))[kSelThreads - 1 - tid];
#pragma unroll
    for (int r = 0; r < kSelCluster; ++r)
      if (r < nranks) {
        hv[0] += q[r].w;
        hv[1] += q[r].z;
        hv[2] += q[r].y;
        hv[3] += q[r].x;
      }
    first_digit();
    // this CTA's candidates, from the cache
    if (mode == 2) {
      for (int j = 0; j < kpt; ++j) {
        bool c = false;
        uint32_t key = 0;
        if (static_cast<int64_t>(tid) * kpt + j < len) {
          bool f;
          load_own(j, key, f);
          c = f && (key >> (32 - kSelTopBits)) == d1;
        }
        append(c, key);
      }
    }
  }
  __syncthreads();
  if (tid < nranks) {
    uint32_t* dst = cluster.map_shared_rank(&info_a[0][0], tid);
    dst[rank * 2 + 0] = np_cta;
    dst[rank * 2 + 1] = s_ncand;
  }
  cluster.sync();  // (A) counts and candidates published; the first-digit counts read
  // every rank has read the gate's histogram: leave it zeroed for the next call
  if (rank == 0 && p.hist_clear)
    for (int b = tid; b < (1 << kSelTopBits); b += kSelThreads) p.hist_clear[b] = 0u;

  uint32_t np_sum = 0, ncand = 0;
  bool over = false;
  for (int r = 0; r < nranks; ++r) {
    if (tid == 0) s_off[r] = ncand;  // where rank r's candidates start in the gathered list
    np_sum += info_a[r][0];
    over = over || info_a[r][1] > static_cast<uint32_t>(kSelOwnCap);
    ncand += info_a[r][1];
  }
  over = over || ncand > static_cast<uint32_t>(kSelAllCap);
  if (tid == 0 && rank == 0 && (static_cast<int64_t>(np_sum) != p.n_prunable || np_sum != np_total))
    raise_error(kErrMaskCount, 1);

  // ---- the low 21 bits of T
  uint32_t thr = 0, need_eq = 0;
  if (mode == 2) {
    uint32_t prefix = d1 << (32 - kSelTopBits), pmask = ((1u << kSelTopBits) - 1u) << (32 - kSelTopBits);
    if (!over) {
      // gather every rank's candidates (four remote loads in flight a thread)
      // and count their next digit; each pass has its own zeroed counts and pick
      __syncthreads();  // s_off written
      for (uint32_t base = 0; base < ncand; base += 4 * kSelThreads) {
        uint32_t v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint32_t idx = base + u * kSelThreads + tid;
          v[u] = 0;
          if (idx < ncand) {
            int r = 0;
            for (int t = 1; t < nranks; ++t)
              if (s_off[t] <= idx) r = t;
            v[u] = cluster.map_shared_rank(own_cand, r)[idx - s_off[r]];
          }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint32_t idx = base + u * kSelThreads + tid;
          if (idx < ncand) {
            all_cand[idx] = v[u];
            atomicAdd(&lhist[0][(v[u] >> 14) & 127u], 1u);
          }
        }
      }
      __syncthreads();
      for (int pass = 0; pass < 3; ++pass) {
        const int shift = 14 - kSelLowBits * pass;
        if (pass > 0) {
          for (uint32_t idx = tid; idx < ncand; idx += kSelThreads) {
            const uint32_t v = all_cand[idx];
            if ((v & pmask) == prefix) atomicAdd(&lhist[pass][(v >> shift) & 127u], 1u);
          }
          __syncthreads();
        }
        if (warp == 0) {
          uint32_t v[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) v[u] = lhist[pass][127 - 4 * lane - u];
          warp_pick_low_digit(v, rem, s_lpick[pass]);
        }
        __syncthreads();
        rem -= s_lpick[pass][1];
        prefix |= s_lpick[pass][0] << shift;
        pmask |= 127u << shift;
      }
    } else {
      // too many candidates: the low bits by cluster-wide passes over the
      // cached keys, the counts merged through distributed shared memory
      for (int pass = 0; pass < 3; ++pass) {
        const int shift = 14 - kSelLowBits * pass;
        if (tid < (1 << kSelLowBits)) hist[tid] = 0;
        __syncthreads();
        for (int j = 0; j < kpt; ++j) {
          if (static_cast<int64_t>(tid) * kpt + j < len) {
            uint32_t key;
            bool f;
            load_own(j, key, f);
            if (f && (key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 127u], 1u);
          }
        }
        cluster.sync();
        if (warp == 0) {
          uint32_t v[4] = {0u, 0u, 0u, 0u};
          for (int r = 0; r < nranks; ++r) {
            const uint32_t* rh = cluster.map_shared_rank(hist, r);
#pragma unroll
            for (int u = 0; u < 4; ++u) v[u] += rh[127 - 4 * lane - u];
          }
          warp_pick_low_digit(v, rem, s_pick);
        }
        __syncthreads();
        rem -= s_pick[1];
        prefix |= s_pick[0] << shift;
        pmask |= 127u << shift;
        cluster.sync();  // every rank has read the remote counts (and s_pick)
      }
    }
    thr = prefix;
    need_eq = rem;  // ties at T to keep
  }

  // ---- this thread's tokens kept outright and its ties at T
  auto classify = [&](int j, bool& ngt, bool& eq) {
    uint32_t key;
    bool f;
    load_own(j, key, f);
    ngt = !f || mode == 1 || (mode == 2 && key > thr);
    eq = f && mode == 2 && key == thr;
  };
  uint32_t n_gt = 0, n_eq = 0;
  for (int j = 0; j < kpt; ++j) {
    if (static_cast<int64_t>(tid) * kpt + j < len) {
      bool ngt, eq;
      classify(j, ngt, eq);
      n_gt += ngt ? 1u : 0u;
      n_eq += eq ? 1u : 0u;
    }
  }
  uint32_t gt_ex, eq_ex, gt_cta, eq_cta;
  if (kpt * kSelThreads < 65536) {
    uint32_t tot;
    const uint32_t ex = block_exclusive_scan(n_eq | (n_gt << 16), warp_sums, &tot);
    gt_ex = ex >> 16;
    eq_ex = ex & 0xffffu;
    gt_cta = tot >> 16;
    eq_cta = tot & 0xffffu;
  } else {
    gt_ex = block_exclusive_scan(n_gt, warp_sums, &gt_cta);
    eq_ex = block_exclusive_scan(n_eq, warp_sums, &eq_cta);
  }
  if (tid < nranks) {
    uint32_t* dst = cluster.map_shared_rank(&info_b[0][0], tid);
    dst[rank * 2 + 0] = gt_cta;
    dst[rank * 2 + 1] = eq_cta;
  }
  cluster.sync();  // (B) the counts are in; no remote access after this

  // cluster-wide prefixes: tokens kept by lower ranks, ties at T in lower ranks
  uint32_t kept_before = 0, eq_before = 0, eq_acc = 0;
  for (int r = 0; r < nranks; ++r) {
    const uint32_t gt_r = info_b[r][0], eq_r = info_b[r][1];
    if (r < rank) {
      kept_before += gt_r + (min(eq_acc + eq_r, need_eq) - min(eq_acc, need_eq));
      eq_before += eq_r;
    }
    eq_acc += eq_r;
  }

  // ---- ordered compaction: this thread's kept tokens in index order
  uint32_t e0 = eq_before + eq_ex;  // ties at T before this thread's tokens (cluster-wide)
  uint32_t pos = kept_before + gt_ex + (min(e0, need_eq) - min(eq_before, need_eq));
  for (int j = 0; j < kpt; ++j) {
    const int64_t i = static_cast<int64_t>(tid) * kpt + j;
    if (i < len) {
      bool ngt, eq;
      classify(j, ngt, eq);
      if (ngt || (eq && e0 < need_eq)) {
        if (pos < p.m) {
          p.out[pos] = static_cast<int32_t>(lo + i);
        } else {
          raise_error(kErrSelectOverflow, 1);
        }
        ++pos;
      }
      if (eq) ++e0;
    }
  }
}

}  // namespace tg

namespace tg {

// ---------------------------------------------------------------------------
// Single-CTA selector for short prompts (n <= kSelSmallMax).  Thread t owns
// the kpt consecutive tokens [t*kpt, (t+1)*kpt).  Keys are loaded coalesced
// (consecutive threads read consecutive tokens) into shared memory laid out
// slot(j) = (j % kpt) * 1025 + j / kpt, so both the loading writes and each
// owner's reads of its own keys spread over the banks.  Four radix passes on
// 8-bit digits count into per-warp histograms (real scores share their
// exponent bits, so one shared histogram would serialise on a few bins); the
// ordered compaction needs one block scan of the packed per-thread
// (kept-above-T, tied-at-T) counts, because each thread's tokens are
// consecutive.
// ---------------------------------------------------------------------------
constexpr int kSelSmallThreads = 1024;
constexpr int kSelSmallWarps = kSelSmallThreads / 32;
constexpr int kSelSmallKpt = 32;
constexpr int kSelSmallMax = kSelSmallThreads * kSelSmallKpt;  // 32768 tokens the CTA can hold
// above this many tokens a cluster of 2048-token slices is faster than one
// CTA (measured on B200: 16K tokens 19.3 us in one CTA, 17.0 us in 8 CTAs;
// 32K 32.7 us vs 21.4 us in 16 CTAs)
constexpr int kSelSmallBest = 4096;
constexpr int kSelSlice = 2048;  // tokens per cluster CTA, until the cluster is at its largest
constexpr int kSelSmallStride = kSelSmallThreads + 1;

__device__ __forceinline__ uint32_t block_exclusive_scan_1024(uint32_t v, uint32_t* warp_sums, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    const uint32_t w = warp_sums[lane];
    uint32_t wx = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, wx, o);
      if (lane >= o) wx += y;
    }
    warp_sums[lane] = wx - w;
    if (lane == 31) warp_sums[32] = wx;
  }
  __syncthreads();
  const uint32_t r = warp_sums[warp] + x - v;
  *total = warp_sums[32];
  __syncthreads();
  return r;
}

// dynamic shared memory: keys [KPT * 1025] uint32, then flags [KPT * 1025] uint8.
// KPT (tokens per thread) is a power of two with KPT * 1024 >= n; vec = 1 when
// scores and mask are 16- and 4-byte aligned (4 tokens per load).
template <int KPT>
__global__ void __launch_bounds__(kSelSmallThreads, 1) k_topk_select_cta(SelectParams p, int vec) {
  pdl_wait();
  pdl_launch_dependents();
  extern __shared__ __align__(16) uint32_t skeys[];
  __shared__ uint32_t whist[kSelSmallWarps][256];
  __shared__ uint32_t warp_sums[33];
  __shared__ uint32_t s_pick[2];
  constexpr int kpt = KPT;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint8_t* sflag = reinterpret_cast<uint8_t*>(skeys + static_cast<size_t>(kpt) * kSelSmallStride);
  const int64_t t0 = static_cast<int64_t>(tid) * kpt;

  // coalesced loads of keys and flags, all of a thread's loads issued before
  // its shared-memory stores
  auto put = [&](int64_t j, float sc, bool f) {
    const int slot = static_cast<int>(j % kpt) * kSelSmallStride + static_cast<int>(j / kpt);
    skeys[slot] = f ? order_key(sc) : 0u;
    sflag[slot] = f ? 1 : 0;
  };
  if (vec) {
    constexpr int V = KPT / 4;  // 16-byte vectors per thread
    float4 sv[V];
    uint32_t mv[V];
    const int64_t n4 = p.n / 4;
#pragma unroll
    for (int u = 0; u < V; ++u) {
      const int64_t v = tid + static_cast<int64_t>(u) * kSelSmallThreads;
      if (v < n4) {
        sv[u] = __ldg(reinterpret_cast<const float4*>(p.scores) + v);
        mv[u] = __ldg(reinterpret_cast<const uint32_t*>(p.prunable) + v);
      }
    }
#pragma unroll
    for (int u = 0; u < V; ++u) {
      const int64_t v = tid + static_cast<int64_t>(u) * kSelSmallThreads;
      if (v < n4) {
        put(4 * v + 0, sv[u].x, (mv[u] & 0xffu) != 0);
        put(4 * v + 1, sv[u].y, (mv[u] & 0xff00u) != 0);
        put(4 * v + 2, sv[u].z, (mv[u] & 0xff0000u) != 0);
        put(4 * v + 3, sv[u].w, (mv[u] & 0xff000000u) != 0);
      }
    }
    for (int64_t j = 4 * n4 + tid; j < p.n; j += kSelSmallThreads) put(j, p.scores[j], p.prunable[j] != 0);
  } else {
    for (int64_t j = tid; j < p.n; j += kSelSmallThreads) put(j, p.scores[j], p.prunable[j] != 0);
  }
  __syncthreads();
  uint32_t fmask = 0;
#pragma unroll
  for (int i = 0; i < kpt; ++i)
    if (t0 + i < p.n && sflag[i * kSelSmallStride + tid]) fmask |= 1u << i;
  uint32_t np_total;
  block_exclusive_scan_1024(__popc(fmask), warp_sums, &np_total);
  if (tid == 0 && static_cast<int64_t>(np_total) != p.n_prunable) raise_error(kErrMaskCount, 2);
  const int64_t kp = min(p.k, static_cast<int64_t>(np_total));
  const int mode = kp <= 0 ? 0 : (kp >= np_total ? 1 : 2);

  uint32_t thr = 0, need_eq = 0;
  if (mode == 2) {
    uint32_t prefix = 0, pmask = 0, remaining = static_cast<uint32_t>(kp);
    for (int pass = 0; pass < 4; ++pass) {
      const int shift = 24 - 8 * pass;
      for (int b = lane; b < 256; b += 32) whist[warp][b] = 0;
      __syncwarp();
#pragma unroll
      for (int i = 0; i < kpt; ++i) {
        const uint32_t key = skeys[i * kSelSmallStride + tid];
        if (((fmask >> i) & 1u) && (key & pmask) == prefix) atomicAdd(&whist[warp][(key >> shift) & 255u], 1u);
      }
      __syncthreads();
      // bin b (counted from the top) summed over the warps by thread b
      uint32_t cnt = 0;
      if (tid < 256) {
#pragma unroll 8
        for (int w = 0; w < kSelSmallWarps; ++w) cnt += whist[w][255 - tid];
      }
      uint32_t tot;
      const uint32_t above = block_exclusive_scan_1024(cnt, warp_sums, &tot);
      if (tid < 256 && above < remaining && remaining <= above + cnt) {
        s_pick[0] = 255u - tid;
        s_pick[1] = above;
      }
      __syncthreads();
      const uint32_t digit = s_pick[0];
      remaining -= s_pick[1];
      prefix |= digit << shift;
      pmask |= 0xffu << shift;
      __syncthreads();  // s_pick and the histograms are rewritten by the next pass
    }
    thr = prefix;
    need_eq = remaining;
  }

  // ordered compaction: per-thread counts and one packed scan (each thread's
  // tokens are consecutive); the kept indices are first placed in shared
  // memory (over the key area) and then written out coalesced
  uint32_t keys[kpt];
#pragma unroll
  for (int i = 0; i < kpt; ++i) keys[i] = skeys[i * kSelSmallStride + tid];
  uint32_t ngt = 0, eq = 0;
#pragma unroll
  for (int i = 0; i < kpt; ++i) {
    if (t0 + i >= p.n) break;
    const bool f = (fmask >> i) & 1u;
    ngt += (!f || mode == 1 || (mode == 2 && keys[i] > thr)) ? 1u : 0u;
    eq += (f && mode == 2 && keys[i] == thr) ? 1u : 0u;
  }
  uint32_t tot;
  const uint32_t ex = block_exclusive_scan_1024((ngt << 16) | eq, warp_sums, &tot);  // (ends with a barrier)
  int32_t* sout = reinterpret_cast<int32_t*>(skeys);  // m <= n <= kpt * 1025 entries
  uint32_t ngt_run = ex >> 16, eq_run = ex & 0xffffu;
#pragma unroll
  for (int i = 0; i < kpt; ++i) {
    const int64_t j = t0 + i;
    if (j >= p.n) break;
    const bool f = (fmask >> i) & 1u;
    const bool g = !f || mode == 1 || (mode == 2 && keys[i] > thr);
    const bool e = f && mode == 2 && keys[i] == thr;
    const bool keep = g || (e && eq_run < need_eq);
    if (keep) {
      const uint32_t pos = ngt_run + min(eq_run, need_eq);
      if (pos < p.m) {
        sout[pos] = static_cast<int32_t>(j);
      } else {
        raise_error(kErrSelectOverflow, 2);
      }
    }
    ngt_run += g ? 1u : 0u;
    eq_run += e ? 1u : 0u;
  }
  __syncthreads();
  const int64_t kept_total = min(static_cast<int64_t>((tot >> 16) + min(tot & 0xffffu, need_eq)), p.m);
  for (int64_t r = tid; r < kept_total; r += kSelSmallThreads) p.out[r] = sout[r];
}

}  // namespace tg

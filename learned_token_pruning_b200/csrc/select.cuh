// Masked top-K selection with stable compaction.
//
// TokenGate keeps S = top-K(b_j) over the prunable (document) tokens plus
// every non-prunable (question) token ("TokenGate and T2Quant: a close
// reading", §4.1 "Top-K selector").  The kept set must come out identical to a
// full stable sort by (score desc, index asc), so the selection runs on
// integer keys that order fp32 scores totally:
//   -0 and +0 map to the same key, NaN maps below -inf, larger score = larger key.
//
// One launch, one thread-block cluster of up to kSelCluster CTAs (the host
// picks the smallest cluster whose slices fit the per-CTA key cache, so short
// prompts run in a single CTA with no cluster-wide barrier).  Each CTA owns a
// contiguous slice of the tokens and, when it fits, keeps its keys in shared
// memory for every pass.  Four 8-bit radix passes find the threshold key T and
// how many ties at T must be kept; the per-pass histograms are merged through
// distributed shared memory.  A last ordered pass writes the kept indices in
// ascending order, breaking ties at T towards the lower index, using one
// exclusive block scan per chunk and cluster-wide prefix counts.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"

namespace tg {

namespace cg = cooperative_groups;

constexpr int kSelCluster = 16;  // 16 needs the non-portable cluster size (the host falls back to 8)
constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / 32;
constexpr size_t kSelCacheBytes = 200 * 1024;  // dynamic smem for the key cache

__device__ __forceinline__ uint32_t order_key(float s) {
  uint32_t b = __float_as_uint(s);
  if ((b & 0x7fffffffu) > 0x7f800000u) return 0u;  // NaN: lowest key
  if (b == 0x80000000u) b = 0u;                     // -0 ranks with +0
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

struct SelectParams {
  const float* scores;
  const uint8_t* prunable;
  int64_t n;
  int64_t n_prunable;
  int64_t k;
  int32_t* out;
  int64_t m;
  int64_t slice;  // tokens per CTA
  int cached;     // 1 if each slice's keys fit the shared-memory cache
};

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

__global__ void __launch_bounds__(kSelThreads, 1) k_topk_select(SelectParams p) {
  pdl_wait();
  pdl_launch_dependents();
  extern __shared__ __align__(16) uint8_t sel_smem[];
  __shared__ uint32_t hist[256];
  __shared__ uint32_t warp_sums[kSelWarps + 1];
  __shared__ uint32_t info[4];      // this CTA's: prunable count, non-prunable count, gt count, eq count
  __shared__ uint32_t s_pick[2];    // chosen digit, keys above the chosen digit (cluster-wide)

  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int nranks = static_cast<int>(cluster.num_blocks());
  const int tid = threadIdx.x;
  const int64_t lo = static_cast<int64_t>(rank) * p.slice;
  const int64_t hi = min(p.n, lo + p.slice);
  const int64_t len = hi > lo ? hi - lo : 0;

  uint32_t* keys = reinterpret_cast<uint32_t*>(sel_smem);
  uint8_t* flags = sel_smem + (p.cached ? p.slice * 4 : 0);

  auto load_key = [&](int64_t i, uint32_t& key, bool& f) {
    if (p.cached) {
      key = keys[i];
      f = flags[i] != 0;
    } else {
      const int64_t j = lo + i;
      f = p.prunable[j] != 0;
      key = f ? order_key(p.scores[j]) : 0u;
    }
  };

  // ---- pass 0: keys, flags and the prunable count of this slice
  uint32_t cnt = 0;
  for (int64_t i = tid; i < len; i += kSelThreads) {
    const int64_t j = lo + i;
    const bool f = p.prunable[j] != 0;
    const uint32_t key = f ? order_key(p.scores[j]) : 0u;
    if (p.cached) {
      keys[i] = key;
      flags[i] = f ? 1 : 0;
    }
    cnt += f ? 1u : 0u;
  }
  uint32_t tot;
  block_exclusive_scan(cnt, warp_sums, &tot);
  if (tid == 0) {
    info[0] = tot;
    info[1] = static_cast<uint32_t>(len) - tot;
  }
  cluster.sync();

  int64_t np_total = 0;
  for (int r = 0; r < nranks; ++r) np_total += *cluster.map_shared_rank(&info[0], r);
  if (tid == 0 && rank == 0 && np_total != p.n_prunable) raise_error(kErrMaskCount, 1);

  const int64_t kp = min(p.k, np_total);
  // mode 0: keep no prunable token; 1: keep all of them; 2: threshold select
  const int mode = kp <= 0 ? 0 : (kp >= np_total ? 1 : 2);

  uint32_t thr = 0, need_eq = 0, local_gt = 0, local_eq = 0;
  if (mode == 2) {
    uint32_t prefix = 0, pmask = 0;
    uint32_t remaining = static_cast<uint32_t>(kp);
    for (int pass = 0; pass < 4; ++pass) {
      const int shift = 24 - 8 * pass;
      if (tid < 256) hist[tid] = 0;
      __syncthreads();
      // warp-aggregated histogram: lanes holding the same digit add once
      // (early digits of real scores crowd into a few bins)
      for (int64_t base = 0; base < len; base += kSelThreads) {
        const int64_t i = base + tid;
        uint32_t key = 0;
        bool f = false;
        if (i < len) load_key(i, key, f);
        const bool valid = f && (key & pmask) == prefix;
        const uint32_t bin = valid ? ((key >> shift) & 255u) : 0xffffffffu;
        const uint32_t peers = __match_any_sync(0xffffffffu, bin);
        if (valid && (threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&hist[bin], __popc(peers));
      }
      cluster.sync();
      // merged histogram, scanned from the top bin down
      uint32_t tot_b = 0, own_b = 0;
      if (tid < 256) {
        const int b = 255 - tid;  // thread 0 holds the top bin
        own_b = hist[b];
        for (int r = 0; r < nranks; ++r) tot_b += cluster.map_shared_rank(hist, r)[b];
      }
      uint32_t total_all;
      const uint32_t above = block_exclusive_scan(tid < 256 ? tot_b : 0u, warp_sums, &total_all);
      if (tid < 256 && above < remaining && remaining <= above + tot_b) {
        s_pick[0] = 255u - tid;
        s_pick[1] = above;
      }
      __syncthreads();
      const uint32_t digit = s_pick[0];
      // keys of this slice strictly above the chosen digit (under the current prefix)
      uint32_t mine = (tid < 256 && (255u - tid) > digit) ? own_b : 0u;
      uint32_t gt_pass;
      block_exclusive_scan(mine, warp_sums, &gt_pass);
      local_gt += gt_pass;
      if (pass == 3) local_eq = hist[digit];
      remaining -= s_pick[1];
      prefix |= digit << shift;
      pmask |= 0xffu << shift;
      cluster.sync();  // every CTA has read the remote histograms
    }
    thr = prefix;
    need_eq = remaining;
  }

  if (tid == 0) {
    info[2] = mode == 1 ? info[0] : local_gt;
    info[3] = local_eq;
  }
  cluster.sync();

  // cluster-wide prefixes for this CTA
  uint32_t eq_before = 0, kept_before = 0;
  {
    uint32_t eq_acc = 0;
    for (int r = 0; r < nranks; ++r) {
      const uint32_t* ri = cluster.map_shared_rank(info, r);
      const uint32_t np_r = ri[1], gt_r = ri[2], eq_r = ri[3];
      const uint32_t tie_keep = eq_acc >= need_eq ? 0u : min(eq_r, need_eq - eq_acc);
      if (r < rank) {
        kept_before += np_r + (mode == 0 ? 0u : gt_r) + tie_keep;
        eq_before += eq_r;
      }
      eq_acc += eq_r;
    }
  }
  cluster.sync();  // remote reads done before any CTA may exit

  // ---- ordered compaction pass
  uint32_t e0 = eq_before;  // ties at T preceding this chunk (cluster-wide)
  uint32_t kept_run = kept_before;
  for (int64_t base = 0; base < len; base += kSelThreads) {
    const int64_t i = base + tid;
    bool ngt = false, eq = false;
    if (i < len) {
      uint32_t key;
      bool f;
      load_key(i, key, f);
      ngt = !f || mode == 1 || (mode == 2 && key > thr);
      eq = f && mode == 2 && key == thr;
    }
    uint32_t chunk_tot;
    const uint32_t ex = block_exclusive_scan((eq ? 1u : 0u) | ((ngt ? 1u : 0u) << 16), warp_sums, &chunk_tot);
    const uint32_t eq_ex = ex & 0xffffu, ngt_ex = ex >> 16;
    const uint32_t g_eq = e0 + eq_ex;
    const bool keep = ngt || (eq && g_eq < need_eq);
    if (keep) {
      const uint32_t pos = kept_run + ngt_ex + (min(g_eq, need_eq) - min(e0, need_eq));
      if (pos < p.m) {
        p.out[pos] = static_cast<int32_t>(lo + i);
      } else {
        raise_error(kErrSelectOverflow, 1);
      }
    }
    const uint32_t eq_tot = chunk_tot & 0xffffu, ngt_tot = chunk_tot >> 16;
    kept_run += ngt_tot + (min(e0 + eq_tot, need_eq) - min(e0, need_eq));
    e0 += eq_tot;
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

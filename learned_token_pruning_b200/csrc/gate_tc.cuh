// Gate scores on the 5th-generation tensor cores ("TokenGate and T2Quant: a
// close reading", §4.1 Gate module):
//     s_j = w2 . SiLU(W1 RMSNorm(h_j) + b1) + b2   for prunable j, 0 otherwise
// with (h_j * w_n) W1^T = h_j (W1 diag(w_n))^T, so the RMSNorm weight is folded
// into W1 on the host side and the row scale 1/rms(h_j) is applied to the
// accumulator in the epilogue.  The hidden states are read from HBM once, and
// into the SM once.
//
// A persistent kernel: one CTA per SM walks the 128-token tiles t = blockIdx.x,
// blockIdx.x + gridDim.x, ...  TMA streams 128x64 tiles of H through a
// kGateHStages-deep ring and BNx64 tiles of W1 through a kGateWStages-deep one
// (128-byte swizzle), both running on across tile boundaries, each fed by its
// own producer thread: the hidden rows come from DRAM, whose latency under a
// full GPU's load needs about 100 KB in flight per SM, while W1 (read by every
// tile) comes from L2.  One thread issues tcgen05.mma (M=128, N=BN, K=16)
// into one of two fp32 TMEM accumulators (2 x BN columns), so the epilogue of
// tile i runs while the MMAs of tile i+1 stream.  Four row-norm warps sum h^2
// of the tile's rows from the same shared-memory stages (one thread per row;
// the swizzle only permutes the 16-byte chunks inside a row's 128-byte line,
// which a sum does not see); a hidden-row stage goes back to its producer
// once the MMAs and these warps have both read it.  Eight epilogue warps, two
// per TMEM lane quarter, each take half of a row's BN accumulator columns,
// apply 1/rms, b1, SiLU and w2, and the halves are added through shared
// memory.  Sum over prunable rows of s^2: per CTA over its tiles in order,
// then over the CTAs in a fixed order by the last CTA to finish
// (deterministic).
//
// Warp roles (480 threads): warp 0 hidden-row producer, warp 1 TMEM allocator
// + MMA issuer, warps 2-5 row norms, warps 6-13 epilogue (warp w reads TMEM
// lanes 32*(w%4)..+31), warp 14 W1 producer.
#pragma once

#include "common.cuh"

namespace tg {

constexpr int kGateBM = 128;
constexpr int kGateBK = 64;
constexpr int kGateThreads = 480;
constexpr int kGateHStages = 7;  // hidden-state ring (from DRAM: the deep one)
constexpr int kGateWStages = 3;  // W1 ring (from L2)

struct GateParams {
  int M, N, K;        // tokens, gate hidden width h, d_model
  const __nv_bfloat16* hidden;
  const float* b1;
  const float* w2;
  float b2;
  float norm_eps;
  const uint8_t* prunable;
  float* scores;
  float* partials;    // [gridDim.x]
  uint32_t* counter;  // zero on entry
  float* sumsq;
  uint32_t* key_hist; // [2048] or null: counts of order_key(s) >> 21 over prunable tokens, zero on entry
};

constexpr int kGateHistBins = 2048;

static_assert(kGateBK == 64, "the MMA loop issues four K = 16 MMAs per 64-column k-step");

// tcgen05.commit to an mbarrier given by its shared-memory address
__device__ __forceinline__ void gate_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

template <int BN>
struct GateCfg {
  static constexpr int kABytes = kGateBM * kGateBK * 2;
  static constexpr int kBBytes = BN * kGateBK * 2;
  static constexpr int kBBox = BN < 128 ? BN : 128;  // rows per W1 TMA box
  static constexpr int kAccCols = BN <= 32 ? 32 : (BN <= 64 ? 64 : (BN <= 128 ? 128 : 256));
  static constexpr int kTmemCols = 2 * kAccCols;   // two accumulators
  static constexpr size_t kSmem = 1024 + kGateHStages * kABytes + kGateWStages * kBBytes + 256 + 2 * BN * 4 +
                                  2 * 2 * 128 * 4 + 64 + kGateHistBins * 4;
};

template <int BN>
__global__ void __launch_bounds__(kGateThreads, 1)
    k_gate_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
              GateParams p) {
  using Cfg = GateCfg<BN>;
  constexpr int HST = kGateHStages, WST = kGateWStages;
  extern __shared__ uint8_t gate_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(gate_smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + HST * Cfg::kABytes;
  uint64_t* hfull = reinterpret_cast<uint64_t*>(sB + WST * Cfg::kBBytes);  // [HST] hidden rows landed
  uint64_t* hempty = hfull + HST;  // [HST] the MMAs and the four row-norm warps have read them
  uint64_t* wfull = hempty + HST;  // [WST] W1 tile landed
  uint64_t* wempty = wfull + WST;  // [WST] the MMAs have read it
  uint64_t* acc_full = wempty + WST;     // [2] accumulator b holds a finished tile
  uint64_t* acc_empty = acc_full + 2;    // [2] the epilogue has read accumulator b (256 arrivals)
  uint64_t* ss_full = acc_empty + 2;     // [2] row sums of squares of the tile in buffer b (128 arrivals)
  uint64_t* ss_free = ss_full + 2;       // [2] the epilogue has read them (256 arrivals)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ss_free + 2);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  float* s_b1 = reinterpret_cast<float*>(smem + HST * Cfg::kABytes + WST * Cfg::kBBytes + 256);
  float* s_w2 = s_b1 + BN;
  float* s_ss = s_w2 + BN;        // [2][128] row sums of h^2 per tile parity
  float* s_half = s_ss + 2 * 128; // [2][128] second-half partial dot products
  float* s_red = s_half + 2 * 128;  // 4 warp partials + broadcast slot
  uint32_t* s_hist = reinterpret_cast<uint32_t*>(s_red + 16);  // [kGateHistBins] this CTA's key histogram

  __shared__ int s_stop[2];  // [tile parity] an epilogue warp saw its wait fail
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int num_k = (p.K + kGateBK - 1) / kGateBK;
  const int tiles = (p.M + kGateBM - 1) / kGateBM;
  // this CTA's tiles: blockIdx.x, blockIdx.x + gridDim.x, ...
  const int my_tiles = blockIdx.x < tiles ? (tiles - 1 - static_cast<int>(blockIdx.x)) / gridDim.x + 1 : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < HST; ++s) {
      mbar_init(&hfull[s], 1);
      mbar_init(&hempty[s], 1 + 4);  // the MMA commit and the four row-norm warps
    }
    for (int s = 0; s < WST; ++s) {
      mbar_init(&wfull[s], 1);
      mbar_init(&wempty[s], 1);  // the MMA commit
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 256);
      mbar_init(&ss_full[b], 128);
      mbar_init(&ss_free[b], 256);
    }
    *abort_flag = 0;
    s_stop[0] = s_stop[1] = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();
  pdl_launch_dependents();

  if (warp == 0 || warp == 14) {
    // ------------------------------------------------------------ TMA producers (run across tiles)
    // Warp 0 streams the hidden rows through the deep ring, warp 14 the W1
    // tiles through the short one, each as far ahead as its own ring allows.
    // Every CTA needs all of W1: walking K from a tile-dependent start spreads
    // the concurrent W1 reads over different L2 lines instead of having every
    // SM hit the same k-tile at once.  (Only the fp32 summation order changes.)
    if (lane == 0) {
      const bool hid = warp == 0;
      prefetch_tmap(hid ? &tmA : &tmB);
      const int nst = hid ? HST : WST;
      int g = 0;  // k-steps issued so far
      for (int i = 0; i < my_tiles && !*abort_flag; ++i) {
        const int tile = blockIdx.x + i * gridDim.x;
        const int kofs = tile % num_k;
        for (int kt = 0; kt < num_k; ++kt, ++g) {
          const int s = g % nst;
          const uint32_t ph = (g / nst) & 1;
          if (!mbar_wait(hid ? &hempty[s] : &wempty[s], ph ^ 1, kErrWaitGemm)) {
            *abort_flag = 1;
            break;
          }
          const int kx = ((kt + kofs) % num_k) * kGateBK;
          if (hid) {
            mbar_arrive_expect_tx(&hfull[s], Cfg::kABytes);
            tma_load_2d(sA + s * Cfg::kABytes, &tmA, &hfull[s], kx, tile * kGateBM);
          } else {
            mbar_arrive_expect_tx(&wfull[s], Cfg::kBBytes);
#pragma unroll
            for (int hb = 0; hb < BN / Cfg::kBBox; ++hb)
              tma_load_2d(sB + s * Cfg::kBBytes + hb * Cfg::kBBox * 128, &tmB, &wfull[s], kx, hb * Cfg::kBBox);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // A barrier check holds back the next tcgen05.mma for its shared-memory
    // round trip, and the tensor core's issue queue is short, so the rings of
    // k-step g + 1 are checked between the second and third MMA of k-step g,
    // while the first two run; the loop keeps its slot and phase counters
    // incrementally and reads the abort flag once per tile.
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kGateBM, BN, false, false);
      // descriptors of stage 0 and barrier addresses, advanced by adding
      // offsets (16-byte units in a descriptor's address field, which cannot
      // carry out of it: shared memory is below 256 KB)
      const uint64_t da0 = sdesc_sw128(smem_u32(sA), 16, 1024), db0 = sdesc_sw128(smem_u32(sB), 16, 1024);
      constexpr uint32_t kAUnits = Cfg::kABytes >> 4, kBUnits = Cfg::kBBytes >> 4;
      const uint32_t hfull_a = smem_u32(hfull), hempty_a = smem_u32(hempty);
      const uint32_t wfull_a = smem_u32(wfull), wempty_a = smem_u32(wempty);
      int sh = 0, sw = 0;          // ring slots of the current k-step
      uint32_t phh = 0, phw = 0;   // and their phases
      uint32_t oa = 0, ob = 0;     // descriptor offsets of those slots
      bool ok = my_tiles == 0 || mbar_wait2(&hfull[0], 0, &wfull[0], 0, kErrWaitGemm);
      for (int i = 0; i < my_tiles && ok; ++i) {
        const int b = i & 1;
        // accumulator b last held tile i - 2: free once its epilogue read it
        if (*abort_flag || (i >= 2 && !mbar_wait(&acc_empty[b], ((i - 2) >> 1) & 1, kErrWaitGemm))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t acc = tmem + b * Cfg::kAccCols;
        const int checks = i == my_tiles - 1 ? num_k - 1 : num_k;  // k-steps followed by another
        for (int kt = 0; kt < num_k; ++kt) {
          const uint64_t da = da0 + oa, db = db0 + ob;
          const int nsh = sh + 1 == HST ? 0 : sh + 1, nsw = sw + 1 == WST ? 0 : sw + 1;
          const uint32_t nphh = nsh == 0 ? phh ^ 1u : phh, nphw = nsw == 0 ? phw ^ 1u : phw;
          umma_ss(acc, da, db, idesc, kt != 0 ? 1u : 0u);
          umma_ss(acc, da + 2, db + 2, idesc, 1u);
          if (kt < checks) {
            const bool rh = mbar_try_wait(hfull_a + nsh * 8, nphh);
            const bool rw = mbar_try_wait(wfull_a + nsw * 8, nphw);
            if (!(rh && rw))
              ok = mbar_wait(&hfull[nsh], nphh, kErrWaitGemm) && mbar_wait(&wfull[nsw], nphw, kErrWaitGemm);
            tc_fence_after();
          }
          umma_ss(acc, da + 4, db + 4, idesc, 1u);
          umma_ss(acc, da + 6, db + 6, idesc, 1u);
          gate_commit(hempty_a + sh * 8);
          gate_commit(wempty_a + sw * 8);
          sh = nsh;
          sw = nsw;
          phh = nphh;
          phw = nphw;
          oa = nsh == 0 ? 0u : oa + kAUnits;
          ob = nsw == 0 ? 0u : ob + kBUnits;
          if (!ok) break;
        }
        if (ok) umma_commit(&acc_full[b]);
      }
      if (!ok) *abort_flag = 1;
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ row norms (one thread per row)
    // Thread `row` reads its row's 128-byte line of each H stage: eight
    // 16-byte chunks, started at a row-dependent chunk so that a quarter-warp
    // touches different bank groups.
    const int row = (warp - 2) * 32 + lane;
    int g = 0;
    for (int i = 0; i < my_tiles; ++i) {
      const int b = i & 1;
      float ss = 0.0f;
      bool ok = true;
      for (int kt = 0; kt < num_k; ++kt, ++g) {
        const int s = g % HST;
        const uint32_t ph = (g / HST) & 1;
        if (*abort_flag || !warp_wait(&hfull[s], ph, kErrWaitGemm)) {
          ok = false;
          break;
        }
        const uint8_t* line = sA + s * Cfg::kABytes + row * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 v = *reinterpret_cast<const uint4*>(line + (((c + row) & 7) << 4));
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            ss = fmaf(bf16_lo(w[t]), bf16_lo(w[t]), ss);
            ss = fmaf(bf16_hi(w[t]), bf16_hi(w[t]), ss);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&hempty[s]);  // release: the reads above come first
      }
      if (!ok) {
        *abort_flag = 1;
        break;
      }
      // s_ss[b] last held tile i - 2: free once its epilogue read it
      if (i >= 2 && !warp_wait(&ss_free[b], ((i - 2) >> 1) & 1, kErrWaitGemm)) {
        *abort_flag = 1;
        break;
      }
      s_ss[b * 128 + row] = ss;
      mbar_arrive(&ss_full[b]);
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 6-13; 14 is a producer)
    const int q = warp & 3;
    const int half = (warp - 6) >> 2;  // 0: columns [0, BN/2), 1: [BN/2, BN)
    const int row = q * 32 + lane;
    const int et = threadIdx.x - 6 * 32;  // 0 .. 255
    const uint32_t t_row = tmem + (static_cast<uint32_t>(q * 32) << 16);
    // columns past h (zero rows of W1 from the TMA bounds fill) contribute nothing
    for (int c = et; c < BN; c += 256) {
      s_b1[c] = (c < p.N && p.b1) ? p.b1[c] : 0.0f;
      s_w2[c] = c < p.N ? p.w2[c] : 0.0f;
    }
    if (p.key_hist)
      for (int c = et; c < kGateHistBins; c += 256) s_hist[c] = 0u;
    asm volatile("bar.sync 1, 256;" ::: "memory");
    float cta_sq = 0.0f;  // this CTA's sum of s^2, tile by tile in order (thread 0 of the group)
    bool stopped = false;
    for (int i = 0; i < my_tiles; ++i) {
      const int b = i & 1;
      const int tile = blockIdx.x + i * gridDim.x;
      const int grow = tile * kGateBM + row;
      const uint32_t ph = (i >> 1) & 1;
      const bool ok = !*abort_flag && warp_wait(&acc_full[b], ph, kErrWaitGemm) && warp_wait(&ss_full[b], ph, kErrWaitGemm);
      // all eight warps take the same decision: a warp whose wait failed sets
      // the tile's stop flag (only ever set) before the barrier, every warp
      // reads it after
      if (!ok && lane == 0) s_stop[b] = 1;
      asm volatile("bar.sync 1, 256;" ::: "memory");
      if (s_stop[b]) {
        *abort_flag = 1;
        stopped = true;
        break;
      }
      const float inv = 1.0f / sqrtf(s_ss[b * 128 + row] / static_cast<float>(p.K) + p.norm_eps);
      mbar_arrive(&ss_free[b]);
      tc_fence_after();
      float acc = 0.0f;
#pragma unroll 1
      for (int c0 = half * (BN / 2); c0 < (half + 1) * (BN / 2); c0 += 32) {
        uint32_t r[32];
        tmem_ld32(t_row + b * Cfg::kAccCols + c0, r);
        tmem_ld_wait();
#pragma unroll
        for (int t = 0; t < 32; ++t) {
          const float uval = fmaf(__uint_as_float(r[t]), inv, s_b1[c0 + t]);
          acc = fmaf(s_w2[c0 + t], __fdividef(uval, 1.0f + __expf(-uval)), acc);
        }
      }
      // accumulator b is read: the MMAs of tile i + 2 may overwrite it
      tc_fence_before();
      mbar_arrive(&acc_empty[b]);
      if (half == 1) s_half[b * 128 + row] = acc;
      asm volatile("bar.sync 1, 256;" ::: "memory");
      if (half == 0) {
        float s = 0.0f;
        bool pr = false;
        if (grow < p.M) {
          pr = p.prunable[grow] != 0;
          s = pr ? (acc + s_half[b * 128 + row]) + p.b2 : 0.0f;
          p.scores[grow] = s;
        }
        if (p.key_hist) {
          // the selector's first radix digit (key bits 31..21) over prunable
          // tokens; lanes holding the same digit add once
          const uint32_t bin = pr ? (order_key(s) >> 21) : 0xffffffffu;
          const uint32_t peers = __match_any_sync(0xffffffffu, bin);
          if (pr && lane == __ffs(peers) - 1) atomicAdd(&s_hist[bin], static_cast<uint32_t>(__popc(peers)));
        }
        // fixed-order reduction of s^2 over this tile's rows, added to the
        // CTA's running sum in tile order
        float sq = s * s;
#pragma unroll
        for (int o = 16; o; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
        if (lane == 0) s_red[q] = sq;
        asm volatile("bar.sync 2, 128;" ::: "memory");
        if (row == 0) cta_sq += (s_red[0] + s_red[1]) + (s_red[2] + s_red[3]);
        asm volatile("bar.sync 2, 128;" ::: "memory");
      }
    }
    if (p.key_hist && !stopped) {
      // this CTA's histogram into the global one (integer adds: the order does not matter)
      asm volatile("bar.sync 1, 256;" ::: "memory");
      for (int c = et; c < kGateHistBins; c += 256)
        if (s_hist[c]) atomicAdd(&p.key_hist[c], s_hist[c]);
    }
    if (half == 0 && !stopped) {
      if (row == 0) {
        p.partials[blockIdx.x] = cta_sq;
        __threadfence();
        const uint32_t prev = atomicAdd(p.counter, 1u);
        s_red[4] = (prev == gridDim.x - 1) ? 1.0f : 0.0f;
      }
      asm volatile("bar.sync 2, 128;" ::: "memory");
      if (s_red[4] != 0.0f) {
        // last CTA: sum the per-CTA partials in a fixed order
        __threadfence();
        float v = 0.0f;
        for (int i = row; i < static_cast<int>(gridDim.x); i += 128) v += __ldcg(p.partials + i);
#pragma unroll
        for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) s_red[q] = v;
        asm volatile("bar.sync 2, 128;" ::: "memory");
        if (row == 0) {
          p.sumsq[0] = (s_red[0] + s_red[1]) + (s_red[2] + s_red[3]);
          *p.counter = 0u;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    __syncwarp();  // the .sync.aligned dealloc needs the whole warp converged
    tmem_dealloc(tmem, Cfg::kTmemCols);
  }
}

}  // namespace tg

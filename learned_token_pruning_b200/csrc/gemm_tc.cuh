// Persistent bf16 GEMM on the 5th-generation tensor cores with fused
// epilogues: C[M][N] = A[M][K] * B[N][K]^T (both operands K-major, the
// nn.Linear layout), fp32 accumulation in tensor memory.
//
// One CTA per SM walks the (128 MH) x BN output tiles (m fastest, so the
// weight block of a column of tiles is fetched from HBM about once).  TMA
// streams MH 128x64 A tiles and a BNx64 B tile (128-byte swizzle) through a
// STAGES-deep shared-memory ring; a single thread issues tcgen05.mma (M=128,
// N=BN, K=16) for each of the MH row halves, which share the B tile.
//   MH = 1: the accumulator is double-buffered in tensor memory (2 x BN
//           columns), so the epilogue drains tile i while tile i+1 runs.
//   MH = 2: a 256 x BN tile reads half as many B bytes per FLOP (the operand
//           feed from L2 is what bounds these GEMMs); its two 128 x BN
//           accumulators fill tensor memory, so the MMAs of tile i+1 wait for
//           the epilogue of tile i.
// A GEMM whose 256-row tiles would leave SMs idle keeps MH = 1.
// Epilogues:
//   kEpiStore     C = acc                                (bf16)
//   kEpiResidual  C = C + acc                            (bf16, in place)
//   kEpiSwiGLU    C[:, f] = SiLU(acc[:, f]) * acc[:, 128 + f]: the B tile of
//                 output block f is the 128 gate rows of those features
//                 followed by their 128 up rows, so the MLP activation is
//                 formed in registers and the [M][2*d_ff] product is never stored.
// Warp roles: warp 0 TMA producer, warp 1 TMEM allocator + MMA issuer, warps
// 2 .. 2+4MH-1 epilogue (warp w reads TMEM lanes 32*(w%4)..+31 of row half
// (w-2)/4).
#pragma once

#include "common.cuh"

namespace tg {

constexpr int kGemmBK = 64;

enum GemmEpilogue { kEpiStore = 0, kEpiResidual = 1, kEpiSwiGLU = 2 };

struct GemmParams {
  int M, N, K;
  int tiles_m, tiles_n;
  __nv_bfloat16* out;
  int64_t ldo;
  int up_row0;  // SwiGLU: first B row of the up block (= d_ff)
};

template <int BN, int STAGES, int MH>
struct GemmCfg {
  static constexpr int kBM = 128 * MH;
  static constexpr int kABytes = kBM * kGemmBK * 2;  // MH boxes of 128 rows
  static constexpr int kBBytes = BN * kGemmBK * 2;
  static constexpr int kBBox = BN < 128 ? BN : 128;  // rows per B TMA box
  static constexpr int kAccCols = BN <= 32 ? 32 : (BN <= 64 ? 64 : (BN <= 128 ? 128 : 256));
  static constexpr int kBufCols = MH * kAccCols;     // one accumulator buffer: every row half
  static constexpr int kBufs = 2 * kBufCols <= 512 ? 2 : 1;
  static constexpr int kTmemCols = kBufs * kBufCols;
  static constexpr int kEpiWarps = 4 * MH;
  static constexpr int kThreads = 64 + 32 * kEpiWarps;
  static constexpr size_t kSmem = 1024 + STAGES * (kABytes + kBBytes) + 256;
};

template <int BN, int STAGES, int EPI, int MH>
__global__ void __launch_bounds__(GemmCfg<BN, STAGES, MH>::kThreads, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, GemmParams p) {
  using Cfg = GemmCfg<BN, STAGES, MH>;
  extern __shared__ uint8_t gemm_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(gemm_smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * Cfg::kABytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + STAGES * Cfg::kBBytes);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;   // [kBufs]
  uint64_t* acc_empty = acc_full + 2;    // [kBufs]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int num_k = (p.K + kGemmBK - 1) / kGemmBK;
  const int tiles = p.tiles_m * p.tiles_n;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < Cfg::kBufs; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], Cfg::kEpiWarps);  // one arrival per epilogue warp
    }
    *abort_flag = 0;
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

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmA);
      prefetch_tmap(&tmB);
      uint32_t it = 0;
      for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
        const int mb = tile % p.tiles_m;
        const int m0 = mb * Cfg::kBM;
        const int nb = tile / p.tiles_m;
        // tiles that share an A row block or a B column block walk K from
        // different starts, so concurrent CTAs do not all read the same L2 lines
        const int kofs = (mb + 7 * nb) % num_k;
        bool ok = true;
        for (int kt = 0; kt < num_k; ++kt, ++it) {
          const uint32_t s = it % STAGES, ph = (it / STAGES) & 1;
          if (*abort_flag || !mbar_wait(&empty[s], ph ^ 1, kErrWaitGemm)) {
            ok = false;
            break;
          }
          const int kx = ((kt + kofs) % num_k) * kGemmBK;
          mbar_arrive_expect_tx(&full[s], Cfg::kABytes + Cfg::kBBytes);
#pragma unroll
          for (int mh = 0; mh < MH; ++mh)
            tma_load_2d(sA + s * Cfg::kABytes + mh * (128 * 128), &tmA, &full[s], kx, m0 + mh * 128);
#pragma unroll
          for (int hb = 0; hb < BN / Cfg::kBBox; ++hb) {
            const int brow = (EPI == kEpiSwiGLU) ? (hb * p.up_row0 + nb * 128) : (nb * BN + hb * Cfg::kBBox);
            tma_load_2d(sB + s * Cfg::kBBytes + hb * Cfg::kBBox * 128, &tmB, &full[s], kx, brow);
          }
        }
        if (!ok) {
          *abort_flag = 1;
          break;
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, BN, false, false);
      uint32_t it = 0;
      int i = 0;
      for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++i) {
        const uint32_t b = i % Cfg::kBufs;
        bool ok = !*abort_flag && mbar_wait(&acc_empty[b], ((i / Cfg::kBufs) & 1) ^ 1, kErrWaitGemm);
        if (ok) {
          tc_fence_after();
          const uint32_t d_tmem = tmem + b * Cfg::kBufCols;
          for (int kt = 0; kt < num_k; ++kt, ++it) {
            const uint32_t s = it % STAGES, ph = (it / STAGES) & 1;
            if (*abort_flag || !mbar_wait(&full[s], ph, kErrWaitGemm)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t a0 = smem_u32(sA + s * Cfg::kABytes);
            const uint32_t b0 = smem_u32(sB + s * Cfg::kBBytes);
#pragma unroll
            for (int mh = 0; mh < MH; ++mh)
#pragma unroll
              for (int kk = 0; kk < kGemmBK / 16; ++kk)
                umma_ss(d_tmem + mh * Cfg::kAccCols, sdesc_sw128(a0 + mh * (128 * 128) + kk * 32, 16, 1024),
                        sdesc_sw128(b0 + kk * 32, 16, 1024), idesc, (kt | kk) != 0 ? 1u : 0u);
            umma_commit(&empty[s]);
          }
        }
        if (!ok) {
          *abort_flag = 1;
          break;
        }
        umma_commit(&acc_full[b]);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue warps
    const int q = warp & 3;
    const int mh = (warp - 2) >> 2;
    const int row = mh * 128 + q * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    int i = 0;
    for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++i) {
      const uint32_t b = i % Cfg::kBufs;
      if (*abort_flag || !warp_wait(&acc_full[b], (i / Cfg::kBufs) & 1, kErrWaitGemm)) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const int grow = (tile % p.tiles_m) * Cfg::kBM + row;
      const int nb = tile / p.tiles_m;
      const uint32_t t_row = tmem + lane_base + b * Cfg::kBufCols + mh * Cfg::kAccCols;
      if (EPI == kEpiStore || EPI == kEpiResidual) {
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 32) {
          uint32_t r[32];
          tmem_ld32(t_row + c0, r);
          tmem_ld_wait();
          const int gcol = nb * BN + c0;
          if (grow < p.M && gcol < p.N) {
            uint4* dst = reinterpret_cast<uint4*>(p.out + static_cast<int64_t>(grow) * p.ldo + gcol);
            uint4 old[4];
            if (EPI == kEpiResidual) {
#pragma unroll
              for (int v = 0; v < 4; ++v) old[v] = dst[v];
            }
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              float add[8] = {0, 0, 0, 0, 0, 0, 0, 0};
              if (EPI == kEpiResidual) {
                const uint32_t ow[4] = {old[v].x, old[v].y, old[v].z, old[v].w};
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                  add[2 * t] = bf16_lo(ow[t]);
                  add[2 * t + 1] = bf16_hi(ow[t]);
                }
              }
              uint4 o;
              o.x = pack_bf16x2(__uint_as_float(r[8 * v + 0]) + add[0], __uint_as_float(r[8 * v + 1]) + add[1]);
              o.y = pack_bf16x2(__uint_as_float(r[8 * v + 2]) + add[2], __uint_as_float(r[8 * v + 3]) + add[3]);
              o.z = pack_bf16x2(__uint_as_float(r[8 * v + 4]) + add[4], __uint_as_float(r[8 * v + 5]) + add[5]);
              o.w = pack_bf16x2(__uint_as_float(r[8 * v + 6]) + add[6], __uint_as_float(r[8 * v + 7]) + add[7]);
              dst[v] = o;
            }
          }
        }
      } else {
#pragma unroll 1
        for (int c0 = 0; c0 < 128; c0 += 32) {
          uint32_t g[32], u[32];
          tmem_ld32(t_row + c0, g);
          tmem_ld32(t_row + 128 + c0, u);
          tmem_ld_wait();
          const int gcol = nb * 128 + c0;
          if (grow < p.M && gcol < p.N) {
            uint4* dst = reinterpret_cast<uint4*>(p.out + static_cast<int64_t>(grow) * p.ldo + gcol);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              float a[8];
#pragma unroll
              for (int t = 0; t < 8; ++t) {
                const float gv = __uint_as_float(g[8 * v + t]);
                a[t] = gv / (1.0f + __expf(-gv)) * __uint_as_float(u[8 * v + t]);
              }
              uint4 o;
              o.x = pack_bf16x2(a[0], a[1]);
              o.y = pack_bf16x2(a[2], a[3]);
              o.z = pack_bf16x2(a[4], a[5]);
              o.w = pack_bf16x2(a[6], a[7]);
              dst[v] = o;
            }
          }
        }
      }
      // this warp's rows of accumulator b are drained: hand it back to the MMA issuer
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[b]);
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

// Epilogue output staging of one warp: its 32 rows x 64 bf16 columns in the
// 128-byte-swizzled layout of a {64, 32} TMA box (row r at 128 r, 16-byte
// chunk c at c ^ (r & 7), so the 32 lanes' row writes spread over the banks),
// written out by one TMA store per 64 columns (rows and columns past the
// tensor's extent are clipped by the copy engine).
__device__ __forceinline__ void stage_wait_free(uint8_t* stage, int lane) {
  if (lane == 0) bulk_wait_read<0>();  // the previous store has read the buffer
  __syncwarp();
}
__device__ __forceinline__ void stage_put(uint8_t* stage, int lane, int chunk, uint4 v) {
  *reinterpret_cast<uint4*>(stage + lane * 128 + ((chunk ^ (lane & 7)) << 4)) = v;
}
__device__ __forceinline__ void stage_store(uint8_t* stage, int lane, const CUtensorMap* map, int col, int row) {
  fence_proxy_async_smem();  // the generic-proxy writes above, before the copy engine reads them
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(map, stage, col, row);
    bulk_commit();
  }
}

// ---------------------------------------------------------------------------
// Pair GEMM: a cluster of two CTAs (two SMs) computes one 256 x 256 output
// tile with the M = 256 pair form of tcgen05.mma.  Each CTA streams its own
// 128 rows of A and its own 128 rows of B (the even CTA the first half of the
// tile's columns, the odd CTA the second; for SwiGLU that is the gate block
// and the up block of the same 128 features), so per SM and 128-column k-step
// the ring carries 64 KB for 128 x 256 x 128 MACs: the operand feed of the
// 256-row single-SM tile, with each SM's accumulator only 128 x 256 fp32 = 256
// tensor memory columns.  Two accumulator buffers therefore fit, and the
// epilogue of tile i overlaps the MMAs of tile i+1.  A k-step of eight MMAs per
// ring barrier (not four) keeps the MMA thread's barrier checks from leaving
// the tensor pipe idle.
// The even CTA's single MMA thread issues every MMA of the pair; its ring
// barrier `full[s]` counts the TMA bytes of both CTAs, and each commit is sent
// to the even and to the odd CTA's barrier in turn (no multicast copies).
// Warp roles as in k_gemm_tc; the eight epilogue warps of each CTA split its
// 128 rows x 256 columns into two column halves per TMEM lane quadrant.
// ---------------------------------------------------------------------------
constexpr int kPairBK = 128;  // K per ring stage: two 64-column (128-byte swizzled) boxes per operand

template <int STAGES>
struct GemmPairCfg {
  static constexpr int kBox = 128 * kGemmBK * 2;     // one 128-row x 64-column box
  static constexpr int kABytes = 2 * kBox;           // this CTA's 128 rows of A, 128 columns of K
  static constexpr int kBBytes = 2 * kBox;           // this CTA's 128 rows of B
  static constexpr int kAccCols = 256;
  static constexpr int kBufs = 2;
  static constexpr int kTmemCols = kBufs * kAccCols;
  static constexpr int kEpiWarps = 8;
  static constexpr int kThreads = 64 + 32 * kEpiWarps;
  static constexpr int kEpiStage = 32 * 128;  // per epilogue warp: 32 rows x 64 bf16 columns, 128-byte swizzle
  static constexpr size_t kSmem = 1024 + STAGES * (kABytes + kBBytes) + kEpiWarps * kEpiStage + 256;
};

template <int STAGES, int EPI>
__global__ void __launch_bounds__(GemmPairCfg<STAGES>::kThreads, 1)
    k_gemm_pair(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmO, GemmParams p) {
  using Cfg = GemmPairCfg<STAGES>;
  extern __shared__ uint8_t gemm_smem_raw[];
  // every CTA of the cluster gets the same dynamic shared-memory offset, so the
  // aligned operand stages sit at the same address in both (the pair MMA reads
  // the peer's operands at the issuing CTA's descriptor addresses)
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(gemm_smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * Cfg::kABytes;
  uint8_t* sEpi = sB + STAGES * Cfg::kBBytes;  // output staging, one 4 KB buffer per epilogue warp
  uint64_t* full = reinterpret_cast<uint64_t*>(sEpi + Cfg::kEpiWarps * Cfg::kEpiStage);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;  // [2]
  uint64_t* acc_empty = acc_full + 2;   // [2], used in the even CTA
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = static_cast<int>(cluster_id_x()), npairs = static_cast<int>(nclusters_x());
  const int num_k = (p.K + kPairBK - 1) / kPairBK;
  const int tiles = p.tiles_m * p.tiles_n;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);   // the even CTA's expect_tx arrival (+ both CTAs' bytes)
      mbar_init(&empty[s], 1);  // one commit of the even CTA's MMA thread
    }
    for (int b = 0; b < Cfg::kBufs; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 2 * Cfg::kEpiWarps);  // every epilogue warp of both CTAs
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, Cfg::kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers exist before any copy or commit targets them
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // no block-wide wait for the previous kernel here: the producer waits after
  // requesting weight boxes (they do not depend on it), the epilogue warps
  // before they read the residual, and the MMA thread touches no global memory
  pdl_launch_dependents();

  int n_my_tiles = 0;
  for (int tile = pair; tile < tiles; tile += npairs) ++n_my_tiles;
  const uint32_t total_it = static_cast<uint32_t>(n_my_tiles) * static_cast<uint32_t>(num_k);

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      prefetch_tmap(&tmA);
      prefetch_tmap(&tmB);
      const uint32_t full0 = map_to_rank(smem_u32(full), 0);  // the even CTA's ring barriers
      // the first ring stages' B boxes (weights, never written by the previous
      // kernel) are requested before waiting for it, so their DRAM latency
      // overlaps its tail; the A boxes follow once it has finished
      const uint32_t n_pre = num_k < STAGES ? static_cast<uint32_t>(num_k) : STAGES;  // first tile's k-steps only
      {
        const int nb = pair / p.tiles_m;
        const int brow = (EPI == kEpiSwiGLU) ? (static_cast<int>(rank) * p.up_row0 + nb * 128)
                                             : (nb * 256 + static_cast<int>(rank) * 128);
        for (uint32_t t = 0; t < n_pre; ++t) {  // fresh barriers: every stage is free
          if (rank == 0) mbar_arrive_expect_tx(&full[t], 2 * (Cfg::kABytes + Cfg::kBBytes));
#pragma unroll
          for (int h = 0; h < 2; ++h)
            tma_load_2d_pair(sB + t * Cfg::kBBytes + h * Cfg::kBox, &tmB, full0 + 8 * t,
                             static_cast<int>(t) * kPairBK + h * kGemmBK, brow);
        }
      }
      pdl_wait();
      uint32_t it = 0;
      bool ok = true;
      for (int tile = pair; tile < tiles && ok; tile += npairs) {
        const int mb = tile % p.tiles_m;
        const int nb = tile / p.tiles_m;
        const int m0 = mb * 256 + static_cast<int>(rank) * 128;
        const int brow = (EPI == kEpiSwiGLU) ? (static_cast<int>(rank) * p.up_row0 + nb * 128)
                                             : (nb * 256 + static_cast<int>(rank) * 128);
        // every tile walks K from 0: concurrent tiles of a row block then start
        // on the same A columns, which the first wave finds in L2 (a per-tile
        // k offset made that first wave a DRAM burst about 1.3 us longer)
        for (int kt = 0; kt < num_k; ++kt, ++it) {
          const uint32_t s = it % STAGES, ph = (it / STAGES) & 1;
          const int kx = kt * kPairBK;
          // the second box of a last, partial k-step may lie past K: the copy
          // engine fills it with zeros, which add nothing to the products
          if (it < n_pre) {  // B already requested, barrier already armed
#pragma unroll
            for (int h = 0; h < 2; ++h)
              tma_load_2d_pair(sA + s * Cfg::kABytes + h * Cfg::kBox, &tmA, full0 + 8 * s, kx + h * kGemmBK, m0);
            continue;
          }
          if (*abort_flag || !mbar_wait(&empty[s], ph ^ 1, kErrWaitGemm)) {
            ok = false;
            break;
          }
          if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * (Cfg::kABytes + Cfg::kBBytes));
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            tma_load_2d_pair(sA + s * Cfg::kABytes + h * Cfg::kBox, &tmA, full0 + 8 * s, kx + h * kGemmBK, m0);
            tma_load_2d_pair(sB + s * Cfg::kBBytes + h * Cfg::kBox, &tmB, full0 + 8 * s, kx + h * kGemmBK, brow);
          }
        }
      }
      if (ok) {
        // the last commits of this CTA's ring have landed before it may exit
        for (uint32_t t = total_it > STAGES ? total_it - STAGES : 0; t < total_it && ok; ++t)
          ok = mbar_wait(&empty[t % STAGES], (t / STAGES) & 1, kErrWaitGemm);
      }
      if (!ok) *abort_flag = 1;
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(256, 256, false, false);
      const uint32_t empty_own = smem_u32(empty), empty_peer = map_to_rank(smem_u32(empty), 1);
      const uint32_t accf_own = smem_u32(acc_full), accf_peer = map_to_rank(smem_u32(acc_full), 1);
      uint32_t it = 0;
      int i = 0;
      bool ok = true;
      for (int tile = pair; tile < tiles; tile += npairs, ++i) {
        const uint32_t b = i % Cfg::kBufs;
        ok = !*abort_flag && mbar_wait_cluster(&acc_empty[b], ((i / Cfg::kBufs) & 1) ^ 1, kErrWaitGemm);
        if (!ok) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + b * Cfg::kAccCols;
        for (int kt = 0; kt < num_k; ++kt, ++it) {
          const uint32_t s = it % STAGES, ph = (it / STAGES) & 1;
          if (*abort_flag || !mbar_wait(&full[s], ph, kErrWaitGemm)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + s * Cfg::kABytes);
          const uint32_t b0 = smem_u32(sB + s * Cfg::kBBytes);
#pragma unroll
          for (int kk = 0; kk < kPairBK / 16; ++kk) {
            const uint32_t off = (kk >> 2) * Cfg::kBox + (kk & 3) * 32;
            umma_ss_pair(d_tmem, sdesc_sw128(a0 + off, 16, 1024), sdesc_sw128(b0 + off, 16, 1024), idesc,
                         (kt | kk) != 0 ? 1u : 0u);
          }
          umma_commit_pair(empty_own + 8 * s);
          umma_commit_pair(empty_peer + 8 * s);
        }
        if (!ok) break;
        umma_commit_pair(accf_own + 8 * b);
        umma_commit_pair(accf_peer + 8 * b);
      }
      if (ok) {
        // both CTAs' epilogues have released the last accumulators (no remote
        // arrival is still on its way to this CTA when it exits)
        for (int t = i > Cfg::kBufs ? i - Cfg::kBufs : 0; t < i && ok; ++t)
          ok = mbar_wait_cluster(&acc_empty[t % Cfg::kBufs], (t / Cfg::kBufs) & 1, kErrWaitGemm);
      }
      if (!ok) *abort_flag = 1;
    }
  } else {
    // ------------------------------------------------------------ epilogue warps (both CTAs)
    const int q = warp & 3;          // TMEM lane quadrant this warp may access
    const int ch = (warp - 2) >> 2;  // column half of the accumulator
    const int row = static_cast<int>(rank) * 128 + q * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    const uint32_t acc_empty0 = map_to_rank(smem_u32(acc_empty), 0);
    uint8_t* stage = sEpi + (warp - 2) * Cfg::kEpiStage;
    pdl_wait();  // the residual and the output may belong to the previous kernel
    int i = 0;
    for (int tile = pair; tile < tiles; tile += npairs, ++i) {
      const uint32_t b = i % Cfg::kBufs;
      const int grow = (tile % p.tiles_m) * 256 + row;
      const int nb = tile / p.tiles_m;
      const int gcol0 = nb * 256 + ch * 128;  // store / residual: this warp's 128 output columns
      uint4 old[EPI == kEpiResidual ? 16 : 1];
      if (EPI == kEpiResidual) {
        // the row's residual is read before the accumulator is ready, so its
        // memory latency hides behind the tile's MMAs
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if (grow < p.M && gcol0 + 32 * c < p.N) {
            const uint4* src = reinterpret_cast<const uint4*>(p.out + static_cast<int64_t>(grow) * p.ldo + gcol0 + 32 * c);
#pragma unroll
            for (int v = 0; v < 4; ++v) old[4 * c + v] = src[v];
          }
        }
      }
      if (*abort_flag || !warp_wait(&acc_full[b], (i / Cfg::kBufs) & 1, kErrWaitGemm)) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t t_row = tmem + lane_base + b * Cfg::kAccCols;
      const int srow0 = (tile % p.tiles_m) * 256 + static_cast<int>(rank) * 128 + q * 32;  // the warp's first row
      if (EPI == kEpiStore || EPI == kEpiResidual) {
#pragma unroll
        for (int c2 = 0; c2 < 4; c2 += 2) {
          uint32_t r[2][32];
          tmem_ld32(t_row + ch * 128 + 32 * c2, r[0]);
          tmem_ld32(t_row + ch * 128 + 32 * (c2 + 1), r[1]);
          tmem_ld_wait();
          stage_wait_free(stage, lane);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int c = c2 + h;
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              float add[8] = {0, 0, 0, 0, 0, 0, 0, 0};
              if (EPI == kEpiResidual) {
                const uint32_t ow[4] = {old[4 * c + v].x, old[4 * c + v].y, old[4 * c + v].z, old[4 * c + v].w};
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                  add[2 * t] = bf16_lo(ow[t]);
                  add[2 * t + 1] = bf16_hi(ow[t]);
                }
              }
              const uint32_t* rr = r[h];
              uint4 o;
              o.x = pack_bf16x2(__uint_as_float(rr[8 * v + 0]) + add[0], __uint_as_float(rr[8 * v + 1]) + add[1]);
              o.y = pack_bf16x2(__uint_as_float(rr[8 * v + 2]) + add[2], __uint_as_float(rr[8 * v + 3]) + add[3]);
              o.z = pack_bf16x2(__uint_as_float(rr[8 * v + 4]) + add[4], __uint_as_float(rr[8 * v + 5]) + add[5]);
              o.w = pack_bf16x2(__uint_as_float(rr[8 * v + 6]) + add[6], __uint_as_float(rr[8 * v + 7]) + add[7]);
              stage_put(stage, lane, 4 * h + v, o);
            }
          }
          stage_store(stage, lane, &tmO, gcol0 + 32 * c2, srow0);
        }
      } else {
        stage_wait_free(stage, lane);
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
          const int c0 = ch * 64 + 32 * h;
          uint32_t g[32], u[32];
          tmem_ld32(t_row + c0, g);
          tmem_ld32(t_row + 128 + c0, u);
          tmem_ld_wait();
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            float a[8];
#pragma unroll
            for (int t = 0; t < 8; ++t) {
              const float gv = __uint_as_float(g[8 * v + t]);
              a[t] = __fdividef(gv, 1.0f + __expf(-gv)) * __uint_as_float(u[8 * v + t]);
            }
            stage_put(stage, lane, 4 * h + v,
                      make_uint4(pack_bf16x2(a[0], a[1]), pack_bf16x2(a[2], a[3]), pack_bf16x2(a[4], a[5]),
                                 pack_bf16x2(a[6], a[7])));
          }
        }
        stage_store(stage, lane, &tmO, nb * 128 + ch * 64, srow0);
      }
      // this warp's part of accumulator b is drained: release it to the even CTA's MMA thread
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty0 + 8 * b);
    }
    if (lane == 0) bulk_wait_all();  // the output stores are complete before the CTA goes away
  }
  tc_fence_before();
  cluster_sync_all();  // neither CTA leaves while the pair still uses its memory
  if (warp == 1) {
    tc_fence_after();
    __syncwarp();
    tmem_dealloc_pair(tmem, Cfg::kTmemCols);
  }
}

}  // namespace tg

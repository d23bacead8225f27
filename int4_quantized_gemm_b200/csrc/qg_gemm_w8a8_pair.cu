// qg_gemm_w8a8_pair.cu -- prefill W8A8 on CTA pairs (tcgen05 cta_group::2).
//
//   Y[m,n] = float(acc[m,n]) * (x_scale[m] * w_scale[n]) + bias[n]
//   acc[m,n] = sum_k Xq[m,k] * Wq[k,n]   (int8 x int8 -> int32, exact)
//
// Page "量化算法的本质", W8A8矩阵乘法 (the fused int32 -> scaled output
// epilogue); page "量化与多精度算子" §四 (int32 accumulation, dequant while the
// result is on chip); page "Ascend C per-channel INT8 GEMM" §5.3-5.4 (K tiles
// prefetched ahead of the MMA, scale at write-back).
//
// The same computation as the one-SM prefill tiles of qg_gemm_w8a8.cu, on
// 256 x 256 output tiles owned by a two-CTA cluster on two SMs.  Per K block
// each CTA stages its own 128 rows of Xq and its own 128 rows of Wq; the even
// CTA issues one M = 256, N = 256 MMA per 32 bytes of K, which reads both CTAs'
// shared memory and writes each CTA's 128 accumulator rows into that CTA's
// tensor memory.  Per SM and 32-byte K step the tensor core then reads 4 KB of
// A and 4 KB of B (a one-SM 128 x 256 tile reads 4 KB and 8 KB), and TMA writes
// 8 KB instead of 12 KB: the shared-memory traffic that bounds the one-SM tiles.
//
// Warps (both CTAs):
//   warp 0      TMA producer of this CTA's two operand halves (ring of stages).
//   warp 1      pair TMEM allocation; in the even CTA the MMA issuer.
//   warps 2..5  epilogue of this CTA's 128 accumulator rows (double-buffered
//               accumulator, so the epilogue of tile i overlaps tile i+1).
// A stage is complete on the even CTA's stage barrier alone: the even CTA's
// producer arrives on it expecting the bytes of both halves, and both CTAs'
// TMA loads (cta_group::2) signal their bytes there, so the MMA issuer waits
// for both halves of the stage on one barrier.  Stage-free and accumulator-
// ready signals are tcgen05.commit arrivals on the barrier of both CTAs;
// accumulator-drained signals of the odd CTA's epilogue reach the even CTA's
// barrier by remote arrive.  Every wait is bounded.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>


#include "qg_device.cuh"
#include "qg_internal.h"
#include "qg_w8a8_common.cuh"

namespace qg {

static __device__ unsigned long long g_status_pair;

unsigned long long read_clear_status_pair(cudaStream_t s) {
  unsigned long long v = 0, z = 0;
  cudaMemcpyFromSymbolAsync(&v, g_status_pair, sizeof(v), 0, cudaMemcpyDeviceToHost, s);
  cudaMemcpyToSymbolAsync(g_status_pair, &z, sizeof(z), 0, cudaMemcpyHostToDevice, s);
  cudaStreamSynchronize(s);
  return v;
}

constexpr int kPairM = 256;   // output rows per pair tile (128 per CTA)
constexpr int kPairN = 256;   // widest pair tile (MMA N; 128 W rows staged per CTA); TMEM slot width
constexpr int kPairThreads = 192;
constexpr uint32_t kPairTmemCols = 2 * kPairN;  // double-buffered int32 accumulator

template <int STAGES>
struct PairSmem {
  static constexpr int kA = 128 * kBK;  // this CTA's 128 rows of Xq per K block
  static constexpr int kB = 128 * kBK;  // room for this CTA's (up to) 128 rows of Wq per K block
  static constexpr int kStage = kA + kB;
  static constexpr int kRing = STAGES * kStage;
  static constexpr int kBars = (2 * STAGES + 5) * 8 + 16;
  static constexpr int kTotal = 1024 + kRing + kBars;
};

template <int STAGES, bool ZP>
__global__ void __launch_bounds__(kPairThreads, 1)
    w8a8_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const W8A8Params p) {
  using L = PairSmem<STAGES>;
  const int pn = p.pair_n, hn = pn / 2;  // tile columns; Wq rows staged per CTA
  const uint32_t idesc = idesc_i8_s32(kPairM, pn);
  const uint32_t stage_tx = (uint32_t)(2 * (L::kA + hn * kBK));  // both CTAs' halves of a stage

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_base = smem_u32(smem_raw);
  const uint32_t base = (raw_base + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw_base);
  const uint32_t sA = base;
  const uint32_t sB = base + STAGES * L::kA;
  const uint32_t bars = base + L::kRing;
  auto full_bar = [&](int s) { return bars + 8u * s; };
  auto empty_bar = [&](int s) { return bars + 8u * (STAGES + s); };
  auto tfull_bar = [&](int b) { return bars + 8u * (2 * STAGES + b); };
  auto tempty_bar = [&](int b) { return bars + 8u * (2 * STAGES + 2 + b); };
  const uint32_t drain_bar = bars + 8u * (2 * STAGES + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + L::kRing + (2 * STAGES + 5) * 8);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  unsigned long long* status = &g_status_pair;
  const uint32_t rank = cluster_ctarank();  // 0: the CTA that issues the pair MMAs
  const bool leader = rank == 0;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);   // even CTA: its producer's arrival (+ both halves' bytes); unused in the odd CTA
      mbar_init(empty_bar(s), 1);  // one pair commit per stage use
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), 1);
      mbar_init(tempty_bar(b), leader ? 8 : 1);  // the epilogue warps of both CTAs
    }
    mbar_init(drain_bar, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  // Both CTAs' barriers exist before either CTA signals the other, and both
  // CTAs have started before the pair allocation.
  cluster_sync();
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), kPairTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_trigger();
  pdl_wait();  // inputs of the preceding kernel are visible from here on

  const int tiles = p.tiles_a * p.tiles_b;
  const int pair = (int)blockIdx.x >> 1, npairs = (int)gridDim.x >> 1;
  const bool scaled = p.out_dtype != QG_I32;
  bool ok = true;

  if (warp == 0) {
    // ---------------- TMA producer: this CTA's halves of each stage ----------------
    if (lane == 0) {
      const uint64_t pol = policy_evict_last();  // X and W tiles are both re-read by other tiles
      int it = 0;
      for (int t = pair; t < tiles && ok; t += npairs) {
        int ta, tb;
        tile_coords(t, p.tiles_a, p.tiles_b, ta, tb);
        const int row_a = ta * kPairM + (int)rank * 128, row_b = tb * pn + (int)rank * hn;
        for (int kb = 0; kb < p.nkb; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          // stage s of use `it` is free in both CTAs (the pair commit of use it - STAGES)
          if (!mbar_wait(empty_bar(s), ph ^ 1u, status, 41)) { ok = false; break; }
          // the even CTA's stage barrier; the odd CTA's bytes may land before
          // the even CTA's arrival (its pending arrival keeps the phase open)
          const uint32_t fb = leader ? full_bar(s) : mapa_shared(full_bar(s), 0);
          if (leader) mbar_arrive_expect_tx(fb, stage_tx);
          if (tma_ok(sA + s * L::kA, kb * kBK, 1, status, 60))
            tma_load_2d_pair_hint(sA + s * L::kA, &tmA, fb, kb * kBK, row_a, pol);
          if (tma_ok(sB + s * L::kB, kb * kBK, 1, status, 61))
            tma_load_2d_pair_hint(sB + s * L::kB, &tmB, fb, kb * kBK, row_b, pol);
        }
      }
      // Wait (bounded) until the loads already issued have landed, so that no
      // copy into this CTA's shared memory outlives it.  The even CTA sees
      // every landed byte of both halves on its stage barriers.  The odd CTA
      // sees its loads only through the stage-free commits of the MMAs that
      // read them (issued after the stage landed); after a normal run those
      // come within the last stages' MMA time, and once one has not come
      // within the wait limit the MMAs have stopped and the loads, issued that
      // long ago, have landed.
      for (int i = it - 1; i >= 0 && i >= it - STAGES; --i) {
        const uint32_t ph = (uint32_t)(i / STAGES) & 1u;
        if (leader) {
          if (!ok) mbar_wait(full_bar(i % STAGES), ph, status, 49);
        } else if (!mbar_wait(empty_bar(i % STAGES), ph, status, 49)) {
          break;
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------- pair MMA issuer (even CTA) ----------------
      int it = 0, tcount = 0;
      bool issued = false;
      for (int t = pair; t < tiles && ok; t += npairs, ++tcount) {
        const int buf = tcount & 1;
        const uint32_t tph = (uint32_t)(tcount >> 1) & 1u;
        if (!mbar_wait_cluster(tempty_bar(buf), tph ^ 1u, status, 42)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(buf * kPairN);
        for (int kb = 0; kb < p.nkb; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if (!mbar_wait_cluster(full_bar(s), ph, status, 43)) { ok = false; break; }
          tc_fence_after();
          const uint64_t da = sdesc_sw128(sA + s * L::kA);
          const uint64_t db = sdesc_sw128(sB + s * L::kB);
#pragma unroll
          for (int k = 0; k < kBK / 32; ++k) mma_i8_pair(d, da + 2u * k, db + 2u * k, idesc, (kb | k) ? 1u : 0u);
          issued = true;
          mma_commit_pair(empty_bar(s), (uint16_t)0x3);
        }
        if (!ok) break;
        mma_commit_pair(tfull_bar(buf), (uint16_t)0x3);
      }
      // On a failure, let every MMA already issued finish before teardown (they
      // read both CTAs' shared memory and write both CTAs' tensor memory).
      if (!ok && issued) {
        mma_commit_pair(drain_bar, (uint16_t)0x1);
        mbar_wait(drain_bar, 0, status, 48);
      }
    }
  } else {
    // ---------------- epilogue: this CTA's 128 rows of each pair tile ----------------
    const int quad = warp & 3;  // TMEM lanes 32*quad .. 32*quad+31
    const int row = quad * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    int tcount = 0;
    for (int t = pair; t < tiles && ok; t += npairs, ++tcount) {
      int ta, tb;
      tile_coords(t, p.tiles_a, p.tiles_b, ta, tb);
      const int buf = tcount & 1;
      const uint32_t tph = (uint32_t)(tcount >> 1) & 1u;
      if (!mbar_wait(tfull_bar(buf), tph, status, 45)) { ok = false; break; }
      tc_fence_after();
      const uint32_t tbase = tmem + lane_addr + (uint32_t)(buf * kPairN);
      const int m = ta * kPairM + (int)rank * 128 + row;
      const float xs = (m < p.M && scaled) ? __ldg(p.x_scale + m) : 0.0f;
      const float xz = (ZP && p.x_zero && m < p.M) ? __ldg(p.x_zero + m) : 0.0f;
      const int32_t xsum = (ZP && p.x_qsum && m < p.M) ? __ldg(p.x_qsum + m) : 0;
      dispatch_act(p.act, [&](auto gelu) {
#pragma unroll 1
      for (int c0 = 0; c0 < pn; c0 += 16) {
        // column scales and bias: the same 16 addresses for the whole warp
        // (broadcast), issued before the TMEM load so their latency overlaps it
        const int n0 = tb * pn + c0;
        float ws[16], bb[16], wz[16];
        int32_t wsum[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int n = min(n0 + j, p.N - 1);
          ws[j] = scaled ? __ldg(p.w_scale + n) : 0.0f;
          bb[j] = p.bias ? __ldg(p.bias + n) : 0.0f;
          wz[j] = (ZP && p.w_zero) ? __ldg(p.w_zero + n) : 0.0f;
          wsum[j] = (ZP && p.w_qsum) ? __ldg(p.w_qsum + n) : 0;
        }
        uint32_t r[16];
        tmem_ld16(tbase + (uint32_t)c0, r);
        tmem_ld_wait();
        if (m < p.M && n0 < p.N) {
          const int nv = min(16, p.N - n0);
          float v[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float a = ZP ? zp_corrected((int32_t)r[j], xz, xsum, wz[j], wsum[j], p.K) : (float)(int32_t)r[j];
            v[j] = fmaf(a, xs * ws[j], bb[j]);
          }
          apply_act_c<decltype(gelu)::value>(v);
          store_row16(p.y, p.out_dtype, (int64_t)m * p.ldy + n0, nv, v, r);
        }
      }
      });
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (leader) mbar_arrive(tempty_bar(buf));
        else mbar_arrive_remote(mapa_shared(tempty_bar(buf), 0));
      }
    }
  }

  // Lanes 1..31 of warps 0 and 1 arrive here while lane 0 may still be in its
  // loop: reconverge before the warp-collective cluster barrier and dealloc.
  __syncwarp();
  tc_fence_before();
  cluster_sync();  // both CTAs: every MMA, remote arrival and TMEM load is done
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem, kPairTmemCols);
  }
}

template <int STAGES, bool ZP>
static qg_status run_w8a8_pair(const CUtensorMap& tmA, const CUtensorMap& tmB, W8A8Params p, cudaStream_t s) {
  using L = PairSmem<STAGES>;
  static_assert(L::kTotal <= 232448, "above the per-block shared memory limit");
  auto kern = w8a8_pair_kernel<STAGES, ZP>;
  static PerDeviceOnce attr;
  static int max_pairs[64] = {};  // clusters of two that fit the device at once (written under attr)
  int cur = 0;  // this call's device's pair count
  qg_status st = attr.run([&](int dev) {
    qg_status r = check_cuda(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kTotal),
                             "cudaFuncSetAttribute(w8a8 pair)");
    if (r != QG_OK) return r;
    LaunchCfg q(2, kPairThreads, L::kTotal, s, 2);
    int n = 0;
    r = check_cuda(cudaOccupancyMaxActiveClusters(&n, kern, &q.cfg), "cudaOccupancyMaxActiveClusters");
    if (r != QG_OK) return r;
    n = n > 0 ? n : sm_count() / 2;
    if (dev >= 0 && dev < 64) max_pairs[dev] = n;
    cur = n;
    return QG_OK;
  });
  if (st != QG_OK) return st;
  if (cur == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cur = (dev >= 0 && dev < 64) ? max_pairs[dev] : sm_count() / 2;
  }
  const int tiles = p.tiles_a * p.tiles_b;
  const int pairs = tiles < cur ? tiles : cur;
  LaunchCfg lc((unsigned)(2 * pairs), kPairThreads, L::kTotal, s, 2);
  return check_cuda(cudaLaunchKernelEx(&lc.cfg, kern, tmA, tmB, p), "w8a8 pair launch");
}

// Tile width of a pair launch: tiles run in waves of `pairs`, each wave as long
// as one tile, about proportional to its width.  Per SM and 32-byte K step a
// tile reads 4 KB of A and 16 * width bytes of B from shared memory for
// 4096 * width MACs, so narrower tiles read more per MAC (+3 % at 240, +7 % at
// 224, +50 % at 128): only 240 and 224 are candidates, taken when waves x width
// saves at least 3 % over 256 columns.  With 256 columns 2048 x 4096 has 128
// tiles on 74 pairs (1.73 waves, so two); at 240 it has 144 tiles in the same
// two waves, each 6 % shorter.
static int pair_tile_n(int tiles_a, int N, int pairs) {
  const int forced = tuning(kTunePairN);
  if (forced >= 128 && forced <= kPairN && forced % 16 == 0) return forced;
  auto cost = [&](int pn) {
    const long tiles = (long)tiles_a * ((N + pn - 1) / pn);
    return (tiles + pairs - 1) / pairs * pn;
  };
  int best = kPairN;
  for (int pn = kPairN - 16; pn >= 224; pn -= 16)
    if (cost(pn) < cost(best)) best = pn;
  return 100 * cost(best) <= 97 * cost(kPairN) ? best : kPairN;
}

// Prefill W8A8 on CTA pairs: A = Xq (M rows), B = Wq (N rows), 256-row tiles of
// pair_n columns.
template <bool ZP>
qg_status launch_w8a8_pair(W8A8Params p, const int8_t* xq, int64_t ldx, const int8_t* wq, int64_t ldw,
                           cudaStream_t s) {
  CUtensorMap tmA, tmB;
  qg_status st;
  p.tiles_a = (p.M + kPairM - 1) / kPairM;
  p.pair_n = pair_tile_n(p.tiles_a, p.N, sm_count() / 2);
  p.tiles_b = (p.N + p.pair_n - 1) / p.pair_n;
  p.splits = 1;
  if ((st = make_tmap_2d(&tmA, xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)p.K, (uint64_t)p.M,
                         (uint64_t)ldx, kBK, 128, CU_TENSOR_MAP_SWIZZLE_128B)) != QG_OK)
    return st;
  if ((st = make_tmap_2d(&tmB, wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)p.K, (uint64_t)p.N,
                         (uint64_t)ldw, kBK, (uint32_t)(p.pair_n / 2), CU_TENSOR_MAP_SWIZZLE_128B)) != QG_OK)
    return st;
  // Six 32 KB stages per CTA; the QG_PAIR_STAGES switch set to 7 selects seven
  // (the most that fits; measured no faster on B200).
  if (tuning(kTunePairStages) == 7) return run_w8a8_pair<7, ZP>(tmA, tmB, p, s);
  return run_w8a8_pair<6, ZP>(tmA, tmB, p, s);
}

template qg_status launch_w8a8_pair<false>(W8A8Params, const int8_t*, int64_t, const int8_t*, int64_t,
                                           cudaStream_t);
template qg_status launch_w8a8_pair<true>(W8A8Params, const int8_t*, int64_t, const int8_t*, int64_t,
                                          cudaStream_t);

}  // namespace qg

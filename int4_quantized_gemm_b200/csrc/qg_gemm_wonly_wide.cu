// qg_gemm_wonly_wide.cu -- weight-only GEMMs (W8A16, W4A16, symmetric W4A16)
// for token batches wider than the decode tiles (M > 64):
//
//   Y[m,n] = w_scale[n] * sum_k X[m,k] * Wq[k,n] + bias[n]                  (W8A16)
//   Y[m,n] = sum_k X[m,k] * (q[k,n] - z[k/64,n]) * s[k/64,n] + bias[n]      (W4A16)
//
// Page "量化与多精度算子" §四 (weights stored as INT8/INT4, dequantized on chip
// before an FP16 contraction; once the batch grows, the dequantization becomes
// the next cost to hide); page "INT4/FP16混合精度GEMM" §3.2/§4.2 ((q - zp) *
// scale, FP16 matmul with FP32 accumulation, FP16 out).
//
// Each CTA owns one tile of 128 weight rows (output columns n, the 128 TMEM
// lanes) and BN = 128 or 256 token rows (the MMA N dimension), so every
// weight is dequantized once per BN tokens instead of once per 16..64 as in the
// decode tiles.  Dataflow per K block of 128:
//   warp 0      TMA: the weight block (int8, or packed int4 + fp16 scale/zero)
//               into a weight ring, and the X block as two 64-K halves into an
//               activation ring of its own (X is BN/16 times the weight bytes).
//   warp 1      owns TMEM; one thread issues the eight tcgen05.mma kind::f16
//               (M = 128, N = BN, K = 16) of the block, A from tensor memory,
//               B = X from shared memory, into one fp32 accumulator.
//   warps 2-9   dequantizers in two groups of four warps (one warp per TMEM
//               lane quadrant); group g takes blocks g, g+2, ... and writes the
//               fp16 A operand of each block into one of four 64-column A
//               stages (tcgen05.st), in natural K order (no reordering of X).
// Dequantizing a block takes a fraction of its MMA time, so two groups keep
// up; shared memory goes to the activation ring instead (three blocks of X in
// flight at BN = 256), which is what bounds the block rate: each block's X
// comes from L2 with about a microsecond of latency.
// With K split across a cluster of S CTAs (S = 2/4/8, when the weight tiles
// alone do not fill the SMs), each CTA finishes 128/S of the tile's rows.  Once
// its MMAs are done a CTA announces at a cluster barrier that its operand rings
// may be overwritten, stages its fp32 partial tile locally 64 token columns
// (one chunk) at a time, and sends each chunk's rows to the CTA that finishes
// them by bulk copies, chunk by chunk as they are staged.  Each chunk lands on
// a barrier of its own, so the owner sums chunk 0 (its own partial and the
// peers', in rank order: deterministic) while later chunks are still in
// flight, and stores the fp16 results straight from registers.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <type_traits>

#include "qg_dequant.cuh"
#include "qg_device.cuh"
#include "qg_internal.h"

namespace qg {

static __device__ unsigned long long g_status_wide;

unsigned long long read_clear_status_wide(cudaStream_t s) {
  unsigned long long v = 0, z = 0;
  cudaMemcpyFromSymbolAsync(&v, g_status_wide, sizeof(v), 0, cudaMemcpyDeviceToHost, s);
  cudaMemcpyToSymbolAsync(g_status_wide, &z, sizeof(z), 0, cudaMemcpyHostToDevice, s);
  cudaStreamSynchronize(s);
  return v;
}

constexpr int kWideKB = 128;        // K per weight block / A stage (64 TMEM columns)
constexpr int kWideGroups = 2;      // dequantizer groups: block it -> group it % 2
constexpr int kWideAStages = 4;     // A stages in tensor memory: block it -> stage it % 4 (owned by group it % 2)
constexpr int kWideConvWarps = 4 * kWideGroups;
constexpr int kWPrefetch = 6;       // weight blocks fetched into L2 ahead of the weight ring
constexpr int kWideThreads = 32 * (2 + kWideConvWarps);

struct WideParams {
  int M, N, K;
  int tiles_a, tiles_b, nkb, splits;
  const float* w_scale;  // W8A16 only
  const float* bias;
  __half* y;
  int64_t ldy;
  int act;       // qg_activation applied to the fp32 value before the fp16 conversion
  int sym;       // W4: two's-complement codes, no zero points
  int static_w;  // no kernel still in flight writes the weights: first weight stages load before the wait
  int tma_y;     // Y is written through tmY (16-byte aligned, row pitch a multiple of 16 bytes)
  int vec_y;     // Y is 16-byte aligned with a row pitch of a multiple of 8 elements (16-byte stores)
};

template <int BN, bool W4, int XSTAGES, int WSTAGES>
struct WideLayout {
  static constexpr int kXStage = BN * 128;              // 64 K of BN fp16 rows: one 128-byte swizzle atom
  static constexpr int kW = W4 ? 128 * 64 : 128 * 128;  // packed int4 rows (64 B) or int8 rows (128 B)
  static constexpr int kSZ = W4 ? 2 * 128 * 2 : 0;      // scale (and zero) tile: [2 groups][128] fp16
  static constexpr int kWStage = kW + 2 * kSZ;
  static constexpr int kXRing = XSTAGES * kXStage;
  static constexpr int kWRing = WSTAGES * kWStage;
  static constexpr int kRing = kXRing + kWRing;
  // Split-K exchange (reusing the rings once the MMAs are done): this CTA's
  // whole fp32 partial tile is staged locally as [BN/64 chunks][128 rows][64]
  // (256-byte rows, 16-byte units XOR-swizzled by row % 16), and the S - 1
  // peers' parts of the rows it finishes arrive as [S-1 slots][chunk][128/S rows][64].
  static constexpr int kChunks = BN / 64;
  static constexpr int kPartial = 128 * BN * 4;         // one CTA's partial tile
  static constexpr int kMaxSplits = BN >= 256 ? 4 : 8;  // what the exchange area below holds
  static constexpr int kStaging = kPartial / kMaxSplits * (kMaxSplits - 1);  // receive area, then staging
  static constexpr int kExchange = kStaging + kPartial;
  static constexpr int kData = kRing > kExchange ? kRing : kExchange;
  static constexpr int kNumBars = 2 * XSTAGES + 2 * WSTAGES + 2 * kWideAStages + 1 + kChunks;
  static constexpr int kBars = kNumBars * 8 + 16;
  static constexpr int kEpi = 2 * 128 * 4;              // w_scale / bias of the rows this CTA finishes
  static constexpr int kTotal = 1024 + kData + kBars + kEpi;
  static constexpr int kTmemCols = 512;
  static_assert(BN + 64 * kWideAStages <= 512, "accumulator + A stages exceed tensor memory");
  static_assert(kWideAStages % kWideGroups == 0, "each A stage belongs to one dequantizer group");
  static_assert(kXStage % 1024 == 0 && kWStage % 1024 == 0, "stages must keep 1024-byte alignment");
  static_assert(WSTAGES % kWideGroups == 0, "each weight stage belongs to one dequantizer group");
  static_assert(XSTAGES % 2 == 0, "a block takes two consecutive activation stages");
  static_assert(kTotal <= 232448, "above the per-block shared memory limit");
};

// Natural-order pairs (k, k+1), (k+2, k+3), (k+4, k+5), (k+6, k+7) from the
// (k, k+4) pair order of u4x8_to_h2x4: four byte permutes.
__device__ __forceinline__ void pairs_k4_to_natural(uint32_t* o) {
  const uint32_t a = __byte_perm(o[0], o[1], 0x5410), b = __byte_perm(o[2], o[3], 0x5410);
  const uint32_t c = __byte_perm(o[0], o[1], 0x7632), d = __byte_perm(o[2], o[3], 0x7632);
  o[0] = a;
  o[1] = b;
  o[2] = c;
  o[3] = d;
}

template <int BN, bool W4, int XSTAGES, int WSTAGES>
__global__ void __launch_bounds__(kWideThreads, 1)
    wonly_wide_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                      const __grid_constant__ CUtensorMap tmS, const __grid_constant__ CUtensorMap tmZ,
                      const __grid_constant__ CUtensorMap tmY, const WideParams p) {
  using L = WideLayout<BN, W4, XSTAGES, WSTAGES>;
  constexpr uint32_t kIdesc = idesc_f16_f32(128, BN);

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_base = smem_u32(smem_raw);
  const uint32_t base = (raw_base + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw_base);
  const uint32_t sX = base;               // activation ring
  const uint32_t sW = base + L::kXRing;   // weight ring
  const uint32_t bars = base + L::kData;
  auto x_full = [&](int s) { return bars + 8u * s; };
  auto x_empty = [&](int s) { return bars + 8u * (XSTAGES + s); };
  auto w_full = [&](int s) { return bars + 8u * (2 * XSTAGES + s); };
  auto w_empty = [&](int s) { return bars + 8u * (2 * XSTAGES + WSTAGES + s); };
  auto a_full = [&](int a) { return bars + 8u * (2 * XSTAGES + 2 * WSTAGES + a); };
  auto a_empty = [&](int a) { return bars + 8u * (2 * XSTAGES + 2 * WSTAGES + kWideAStages + a); };
  const uint32_t d_full = bars + 8u * (2 * XSTAGES + 2 * WSTAGES + 2 * kWideAStages);
  // split-K: the peers' rows of chunk k (64 token columns) have landed
  auto recv_bar = [&](int k) { return bars + 8u * (2 * XSTAGES + 2 * WSTAGES + 2 * kWideAStages + 1 + k); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + L::kData + L::kNumBars * 8);
  float* sWs = reinterpret_cast<float*>(gbase + L::kData + L::kBars);  // [128]
  float* sBias = sWs + 128;                                            // [128]
  auto stage_x = [&](int s) { return sX + (uint32_t)(s * L::kXStage); };
  auto stage_w = [&](int s) { return sW + (uint32_t)(s * L::kWStage); };
  auto stage_sc = [&](int s) { return sW + (uint32_t)(s * L::kWStage + L::kW); };
  auto stage_ze = [&](int s) { return sW + (uint32_t)(s * L::kWStage + L::kW + L::kSZ); };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  unsigned long long* status = &g_status_wide;

  // one work unit per CTA: (weight tile, token tile, K split)
  const int S = p.splits;
  const int tile = blockIdx.x / S;
  const int split = blockIdx.x % S;
  const int ta = tile % p.tiles_a;  // weight rows (output columns n)
  const int tb = tile / p.tiles_a;  // token rows m
  const int kb0 = split * p.nkb / S, kb1 = (split + 1) * p.nkb / S;
  const int nblk = kb1 - kb0;
  const int rows = 128 / S;         // rows of the tile this CTA finishes (split-K)

  const uint64_t pol_w = policy_evict_first();
  const uint64_t pol_x = policy_evict_last();
  auto load_w = [&](int s, int kb) {
    mbar_arrive_expect_tx(w_full(s), (uint32_t)(L::kW + (W4 ? (p.sym ? 1 : 2) * L::kSZ : 0)));
    if (W4) {
      if (tma_ok(stage_w(s), kb * (kWideKB / 2), 1, status, 60))
        tma_load_2d_hint(stage_w(s), &tmW, w_full(s), kb * (kWideKB / 2), ta * 128, pol_w);
      if (tma_ok(stage_sc(s), ta * 128, 2, status, 61))
        tma_load_2d_hint(stage_sc(s), &tmS, w_full(s), ta * 128, kb * 2, pol_w);
      if (!p.sym && tma_ok(stage_ze(s), ta * 128, 2, status, 62))
        tma_load_2d_hint(stage_ze(s), &tmZ, w_full(s), ta * 128, kb * 2, pol_w);
    } else {
      if (tma_ok(stage_w(s), kb * kWideKB, 1, status, 63))
        tma_load_2d_hint(stage_w(s), &tmW, w_full(s), kb * kWideKB, ta * 128, pol_w);
    }
  };
  // weight block kb towards L2 only (the ring's later load then hits L2)
  auto prefetch_w = [&](int kb) {
    if (W4) {
      if (tma_ok(0u, kb * (kWideKB / 2), 1, status, 64)) tma_prefetch_l2_2d(&tmW, kb * (kWideKB / 2), ta * 128);
      if (tma_ok(0u, ta * 128, 2, status, 65)) tma_prefetch_l2_2d(&tmS, ta * 128, kb * 2);
      if (!p.sym && tma_ok(0u, ta * 128, 2, status, 66)) tma_prefetch_l2_2d(&tmZ, ta * 128, kb * 2);
    } else {
      if (tma_ok(0u, kb * kWideKB, 1, status, 67)) tma_prefetch_l2_2d(&tmW, kb * kWideKB, ta * 128);
    }
  };
  auto load_x = [&](int s, int kb, int half) {
    mbar_arrive_expect_tx(x_full(s), (uint32_t)L::kXStage);
    if (tma_ok(stage_x(s), kb * kWideKB + 64 * half, 2, status, 68))
      tma_load_2d_hint(stage_x(s), &tmX, x_full(s), kb * kWideKB + 64 * half, tb * BN, pol_x);
  };
  int npre = 0;  // weight stages issued before the wait on the preceding kernel

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < XSTAGES; ++s) {
      mbar_init(x_full(s), 1);
      mbar_init(x_empty(s), 1);  // MMA commit
    }
    for (int s = 0; s < WSTAGES; ++s) {
      mbar_init(w_full(s), 1);
      mbar_init(w_empty(s), 4);  // the four warps of the group that dequantized it
    }
    for (int a = 0; a < kWideAStages; ++a) {
      mbar_init(a_full(a), 4);   // the four warps of the group that dequantized into it
      mbar_init(a_empty(a), 1);  // MMA commit
    }
    mbar_init(d_full, 1);
    for (int k = 0; k < L::kChunks; ++k) {
      mbar_init(recv_bar(k), 1);
      // armed at once: the S - 1 peers' parts of chunk k complete it; bytes may
      // land before or after this (the phase needs the arrival as well)
      if (S > 1) mbar_arrive_expect_tx(recv_bar(k), (uint32_t)((S - 1) * rows * 64 * 4));
    }
    fence_mbar_init();
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmW);
    if (W4) {
      tma_prefetch_desc(&tmS);
      if (!p.sym) tma_prefetch_desc(&tmZ);
    }
    if (p.static_w) {
      npre = min(WSTAGES, nblk);
      for (int i = 0; i < npre; ++i) load_w(i, kb0 + i);
    }
    // The weight ring is short (shared memory goes to the activation ring), so
    // weight blocks are fetched into L2 kWPrefetch blocks ahead of it: the ring
    // then waits on L2, not on HBM.  Safe before the wait on the preceding
    // kernel (L2 is the point of coherence).
    for (int i = npre; i < min(npre + kWPrefetch, nblk); ++i) prefetch_w(kb0 + i);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_trigger();
  // Inputs of the preceding kernel are visible after the wait.  With static
  // weights the dequantizer warps skip it: they read only weights (codes,
  // scales, zero points, w_scale, bias), which no kernel in flight writes; X
  // reaches the MMAs through the producer, which waits, and the epilogue's
  // stores follow those MMAs.
  if (!p.static_w || warp < 2) pdl_wait();

  bool ok = true;
  // Split-K tail of the dequantizer warps (kS = S CTAs per cluster, rows =
  // 128 / kS rows finished here).  Group g owns token chunks [g C/2, (g+1) C/2)
  // (C = BN / 64) and handles them end to end:
  //  1. cluster barrier arrive: this CTA's MMAs are done, its rings may be
  //     overwritten by the peers' rows;
  //  2. per chunk: TMEM -> registers -> local staging [chunk][128 rows][64]
  //     (fp32, 16-byte units XOR-swizzled by row % 16), then one bulk copy per
  //     (warp, owner) of the warp's rows that another CTA finishes (the first
  //     copy waits for the barrier: every peer's rings are free);
  //  3. per chunk: wait for the peers' rows, sum the kS partials in rank order,
  //     scale, bias, activation, fp16 stores;
  //  4. cluster barrier arrive: all rows of this CTA have landed.
  auto splitk_tail = [&](auto kS_, bool ok_t, int grp, int quad, int gt, int c_lo, uint32_t lane_addr) {
    constexpr int kS = decltype(kS_)::value;
    constexpr int kRows = 128 / kS;
    constexpr int kGroupChunks = L::kChunks / kWideGroups;
    const int rank = (int)cluster_ctarank();
    const int r0 = rank * kRows;
    const int row = quad * 32 + lane;
    cluster_arrive_relaxed();  // (1)
    bool waited = false;
#pragma unroll 1
    for (int ci = 0; ci < kGroupChunks; ++ci) {
      const int k = grp * kGroupChunks + ci;
      if (ok_t) {
        uint32_t v[2][32];
        tmem_ld32(tmem + lane_addr + (uint32_t)(c_lo + 64 * ci), v[0]);
        tmem_ld32(tmem + lane_addr + (uint32_t)(c_lo + 64 * ci + 32), v[1]);
        tmem_ld_wait();
        uint8_t* srow = gbase + L::kStaging + (k * 128 + row) * 256;
        // debug library: the staged row lies in the exchange area
        if (dcheck(in_area(L::kStaging + (k * 128 + row) * 256, 256, L::kExchange), status, 70)) {
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            const uint32_t* q = &v[u >> 3][(u & 7) * 4];
            *reinterpret_cast<uint4*>(srow + ((u ^ (row & 15)) << 4)) = make_uint4(q[0], q[1], q[2], q[3]);
          }
        }
        fence_proxy_async_smem();  // the staging writes -> the bulk copies
      }
      __syncwarp();
      if (!waited) {
        cluster_wait();  // (1) complete: every CTA's rings are free
        waited = true;
      }
      if (ok_t && lane == 0) {
        constexpr int kSeg = kRows < 32 ? kRows : 32;  // rows per copy: one owner each
#pragma unroll
        for (int r = quad * 32; r < quad * 32 + 32; r += kSeg) {
          const int owner = r / kRows;
          if (owner == rank) continue;
          const int slot = rank < owner ? rank : rank - 1;
          const uint32_t src = base + (uint32_t)(L::kStaging + (k * 128 + r) * 256);
          const uint32_t dst = base + (uint32_t)(((slot * L::kChunks + k) * kRows + r % kRows) * 256);
          // debug library: the rows land in the owner's receive area, before its staging
          if (dcheck(in_area(((slot * L::kChunks + k) * kRows + r % kRows) * 256, kSeg * 256, L::kStaging), status,
                     71))
            bulk_copy_to_cluster(mapa_shared(dst, (uint32_t)owner), src, (uint32_t)(kSeg * 256),
                                 mapa_shared(recv_bar(k), (uint32_t)owner));
        }
      }
    }
    // the group's own rows are staged (barrier ids 2 and 3: one per group)
    if (grp == 0) named_barrier(2, 128);
    else named_barrier(3, 128);
    // (3): each task sums 8 consecutive rows x 4 tokens (one 16-byte unit of
    // 8 rows) over the kS partials, in rank order, and writes 4 runs of 8 fp16
    // outputs (one 16-byte store each where Y allows).  A chunk has kRows / 8 x
    // 16 tasks; the group's threads take the tasks of its chunks in order, so
    // with one task per thread the chunks are reduced side by side.
    constexpr int kTasks = kRows / 8 * 16;
    const float* sws = sWs + grp * 64;
    const float* sbi = sBias + grp * 64;
    dispatch_act(p.act, [&](auto gelu) {
#pragma unroll 1
      for (int t = gt; t < kGroupChunks * kTasks; t += 128) {
        const int ci = t / kTasks, task = t % kTasks;
        const int k = grp * kGroupChunks + ci;
        const int c4 = task & 15, rg = task >> 4;  // 16-byte unit (4 tokens), group of 8 rows
        ok_t = mbar_wait_cluster(recv_bar(k), 0, status, 49) && ok_t;
        const int lr0 = rg * 8;
        const int n0 = ta * 128 + r0 + lr0;
        if (!ok_t || n0 >= p.N) continue;
        float acc[8][4];
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          const int lr = lr0 + r, trow = r0 + lr;
          const int unit = (c4 ^ (trow & 15)) << 4;
          float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
          for (int q = 0; q < kS; ++q) {
            const int off = q == rank ? L::kStaging + (k * 128 + trow) * 256
                                      : (((q < rank ? q : q - 1) * L::kChunks + k) * kRows + lr) * 256;
            // debug library: each read lies in the exchange area
            const bool rd_ok = dcheck(in_area(off + unit, 16, L::kExchange), status, 72);
            const float4 v =
                rd_ok ? *reinterpret_cast<const float4*>(gbase + off + unit) : make_float4(0.f, 0.f, 0.f, 0.f);
            if (q == 0) {
              a = v;
            } else {
              a.x += v.x;
              a.y += v.y;
              a.z += v.z;
              a.w += v.w;
            }
          }
          const float sc = sws[lr], b = sbi[lr];
          acc[r][0] = fmaf(a.x, sc, b);
          acc[r][1] = fmaf(a.y, sc, b);
          acc[r][2] = fmaf(a.z, sc, b);
          acc[r][3] = fmaf(a.w, sc, b);
          apply_act_c<decltype(gelu)::value>(acc[r]);
        }
        const int m0 = tb * BN + 64 * k + 4 * c4;
        const bool vec = p.vec_y && n0 + 8 <= p.N;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (m0 + j >= p.M) break;
          __half* yrow = p.y + (int64_t)(m0 + j) * p.ldy + n0;
          if (vec) {
            uint32_t w[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              const __half2 pr = __floats2half2_rn(acc[2 * h][j], acc[2 * h + 1][j]);
              w[h] = *reinterpret_cast<const uint32_t*>(&pr);
            }
            *reinterpret_cast<uint4*>(yrow) = make_uint4(w[0], w[1], w[2], w[3]);
          } else {
#pragma unroll
            for (int r = 0; r < 8; ++r)
              if (n0 + r < p.N) yrow[r] = __float2half_rn(acc[r][j]);
          }
        }
      }
    });
    cluster_arrive_relaxed();  // (4)
  };
  if (warp == 0) {
    // ---------------- TMA producers ----------------
    // lane 0 streams the weight blocks, lane 1 the activation halves: each
    // ring runs ahead as far as its own free stages allow (the weight ring is
    // short, and must not hold back the activation loads).
    if (lane == 0) {
      int nw = npre;  // weight loads issued
      for (int it = npre; it < nblk; ++it) {
        const int kb = kb0 + it, s = it % WSTAGES;
        if (!mbar_wait(w_empty(s), ((uint32_t)(it / WSTAGES) & 1u) ^ 1u, status, 41)) { ok = false; break; }
        load_w(s, kb);
        ++nw;
        if (it + kWPrefetch < nblk) prefetch_w(kb + kWPrefetch);
      }
      // wait (bounded) for every issued load, so that no copy into this CTA's
      // shared memory outlives it; after a normal run each wait is one poll
      for (int i = nw - 1; i >= 0 && i >= nw - WSTAGES; --i)
        mbar_wait(w_full(i % WSTAGES), (uint32_t)(i / WSTAGES) & 1u, status, 43);
    } else if (lane == 1) {
      int nx = 0;  // activation loads issued
      for (int j = 0; j < 2 * nblk; ++j) {
        const int s = j % XSTAGES;
        if (!mbar_wait(x_empty(s), ((uint32_t)(j / XSTAGES) & 1u) ^ 1u, status, 42)) { ok = false; break; }
        load_x(s, kb0 + j / 2, j & 1);
        ++nx;
      }
      for (int i = nx - 1; i >= 0 && i >= nx - XSTAGES; --i)
        mbar_wait(x_full(i % XSTAGES), (uint32_t)(i / XSTAGES) & 1u, status, 43);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      for (int it = 0; it < nblk; ++it) {
        const int a = it % kWideAStages;
        const int j0 = 2 * it, j1 = 2 * it + 1;
        const int xs0 = j0 % XSTAGES, xs1 = j1 % XSTAGES;
        if (!mbar_wait(a_full(a), (uint32_t)(it / kWideAStages) & 1u, status, 44)) { ok = false; break; }
        if (!mbar_wait(x_full(xs0), (uint32_t)(j0 / XSTAGES) & 1u, status, 45)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a_col = tmem + (uint32_t)(BN + 64 * a);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          mma_f16_ts(tmem, a_col + 8u * j, sdesc_sw128(stage_x(xs0) + (uint32_t)(j * 32)), kIdesc,
                     (it > 0 || j > 0) ? 1u : 0u);
        mma_commit(x_empty(xs0));  // the first half of the block's X is free once these four are done
        if (!mbar_wait(x_full(xs1), (uint32_t)(j1 / XSTAGES) & 1u, status, 45)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int j = 4; j < 8; ++j)
          mma_f16_ts(tmem, a_col + 8u * j, sdesc_sw128(stage_x(xs1) + (uint32_t)((j - 4) * 32)), kIdesc, 1u);
        mma_commit(a_empty(a));
        mma_commit(x_empty(xs1));
      }
      if (ok) mma_commit(d_full);
    }
  } else {
    // ---------------- dequantizers, then epilogue ----------------
    const int cw = warp - 2;                   // 0..7
    const int grp = cw >> 2;                   // group: blocks grp, grp + 2, ...
    const int quad = warp & 3;                 // TMEM lane quadrant this warp may access
    const int row = quad * 32 + lane;          // TMEM lane = weight row within the tile
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    // split-K: scale and bias of the rows this CTA finishes, fetched while the
    // mainloop runs; one copy per group (rows <= 64), read by that group only
    const int gt0 = (cw & 3) * 32 + lane;
    if (S > 1 && gt0 < rows) {
      const int nn = ta * 128 + (int)cluster_ctarank() * rows + gt0;
      sWs[grp * 64 + gt0] = (!W4 && nn < p.N) ? __ldg(p.w_scale + nn) : 1.0f;
      sBias[grp * 64 + gt0] = (p.bias && nn < p.N) ? __ldg(p.bias + nn) : 0.0f;
    }
    for (int it = grp; it < nblk && ok; it += kWideGroups) {
      const int s = it % WSTAGES;
      const int a = it % kWideAStages;
      if (!mbar_wait(w_full(s), (uint32_t)(it / WSTAGES) & 1u, status, 46)) { ok = false; break; }
      if (!mbar_wait(a_empty(a), ((uint32_t)(it / kWideAStages) & 1u) ^ 1u, status, 47)) { ok = false; break; }
      tc_fence_after();
      const uint32_t dst = tmem + lane_addr + (uint32_t)(BN + 64 * a);
      if (W4) {
        // packed row: 64 bytes, 64-byte swizzle (16-byte chunk c at c ^ ((row >> 1) & 3));
        // chunks 0-1 hold quantization group 0 of the block, 2-3 group 1
        const uint8_t* wrow = gbase + (stage_w(s) - base) + row * 64;
        const uint32_t m_lo = p.sym ? 0x64086408u : 0x64006400u;  // magic (+ nibble sign bits)
        const uint32_t m_hi = p.sym ? 0x64806480u : 0x64006400u;
        const __half* sc = reinterpret_cast<const __half*>(gbase + (stage_sc(s) - base));
        const __half* ze = reinterpret_cast<const __half*>(gbase + (stage_ze(s) - base));
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          const uint32_t zb = p.sym ? 0x4800u : (uint32_t)__half_as_ushort(ze[g * 128 + row]);  // 8.0 if sym
          uint32_t s2, c_lo, c_hi;
          u4_group_consts(__half_as_ushort(sc[g * 128 + row]), zb, s2, c_lo, c_hi);
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            const int chunk = 2 * g + cc;
            const uint4 v = *reinterpret_cast<const uint4*>(wrow + ((chunk ^ ((row >> 1) & 3)) << 4));
            const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
            uint32_t r[16];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              u4x8_to_h2x4(wv[i], s2, c_lo, c_hi, m_lo, m_hi, r + 4 * i);
              pairs_k4_to_natural(r + 4 * i);
            }
            tmem_st16(dst + 16 * chunk, r);
          }
        }
      } else {
        // int8 row: 128 bytes, 128-byte swizzle (chunk c at c ^ (row & 7))
        const uint8_t* wrow = gbase + (stage_w(s) - base) + row * 128;
#pragma unroll
        for (int c2 = 0; c2 < 4; ++c2) {
          uint32_t r[16];
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            const int chunk = 2 * c2 + cc;
            const uint4 v = *reinterpret_cast<const uint4*>(wrow + ((chunk ^ (row & 7)) << 4));
            const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) i8x4_to_h2x2(wv[i], r[8 * cc + 2 * i], r[8 * cc + 2 * i + 1]);
          }
          tmem_st16(dst + 16 * c2, r);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(a_full(a));
        mbar_arrive(w_empty(s));
      }
    }
    // epilogue: lane = output column n, accumulator columns = token rows m;
    // group g handles accumulator columns [g BN/4, (g+1) BN/4)
    ok = ok && mbar_wait(d_full, 0, status, 48);
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;  // warp-uniform for the .aligned TMEM loads
    if (ok) tc_fence_after();
    constexpr int kCols = BN / kWideGroups;
    const int c_lo = grp * kCols;
    if (S == 1) {
     if (ok) {
      const int n = ta * 128 + row;
      const bool nvalid = n < p.N;
      const float my_ws = (!W4 && nvalid) ? __ldg(p.w_scale + n) : 1.0f;
      const float my_b = (nvalid && p.bias) ? __ldg(p.bias + n) : 0.0f;
      // The fp16 tile [BN tokens][128 columns] is assembled in the (idle)
      // operand ring and written by one TMA store; without tmY, element stores.
      __half* tile = reinterpret_cast<__half*>(gbase);
      // 64 accumulator columns per tensor-memory round trip (two loads, one wait)
      dispatch_act(p.act, [&](auto gelu) {
#pragma unroll 1
      for (int c0 = c_lo; c0 < c_lo + kCols; c0 += 64) {
        uint32_t v[2][32];
        tmem_ld32(tmem + lane_addr + (uint32_t)c0, v[0]);
        tmem_ld32(tmem + lane_addr + (uint32_t)(c0 + 32), v[1]);
        tmem_ld_wait();
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float f[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) f[j] = fmaf(__uint_as_float(v[h][j]), my_ws, my_b);
          apply_act_c<decltype(gelu)::value>(f);
          if (p.tma_y) {
#pragma unroll
            for (int j = 0; j < 32; ++j) tile[(c0 + 32 * h + j) * 128 + row] = __float2half_rn(f[j]);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int m = tb * BN + c0 + 32 * h + j;
              if (nvalid && m < p.M) p.y[(int64_t)m * p.ldy + n] = __float2half_rn(f[j]);
            }
          }
        }
      }
      });
     }
      if (p.tma_y) {
        // every dequantizer warp gets here (also after a failed wait), then one
        // thread stores the tile
        fence_proxy_async_smem();            // the tile's generic writes -> the TMA store
        named_barrier(1, 32 * kWideConvWarps);
        if (cw == 0 && lane == 0 && ok) {
          if (tma_ok(smem_u32(reinterpret_cast<__half*>(gbase)), ta * 128, 2, status, 69))
            tma_store_2d(&tmY, smem_u32(reinterpret_cast<__half*>(gbase)), ta * 128, tb * BN);
          tma_store_commit();
          tma_store_wait_all();
        }
      }
    }
    if (S == 2) splitk_tail(std::integral_constant<int, 2>{}, ok, grp, quad, gt0, c_lo, lane_addr);
    else if (S == 4) splitk_tail(std::integral_constant<int, 4>{}, ok, grp, quad, gt0, c_lo, lane_addr);
    else if (S == 8 && L::kMaxSplits >= 8)
      splitk_tail(std::integral_constant<int, L::kMaxSplits>{}, ok, grp, quad, gt0, c_lo, lane_addr);
  }
  if (S > 1 && warp < 2) {
    // the producer and the MMA warps take part in the two cluster barriers of
    // the split-K tail and have nothing else to do there
    cluster_arrive_relaxed();
    cluster_wait();
    cluster_arrive_relaxed();
  }
  // Leave only once every CTA of the cluster holds all its rows: until then a
  // peer may still be copying out of this CTA's staging area.
  if (S > 1) cluster_wait();
  tc_fence_before();
  cta_barrier_all();  // every thread of every role is done with TMEM and shared memory
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
template <int BN, bool W4, int XSTAGES, int WSTAGES>
static qg_status run_wide(const CUtensorMap& tmX, const CUtensorMap& tmW, const CUtensorMap& tmS,
                          const CUtensorMap& tmZ, const CUtensorMap& tmY, const WideParams& p, cudaStream_t s) {
  using L = WideLayout<BN, W4, XSTAGES, WSTAGES>;
  auto kern = wonly_wide_kernel<BN, W4, XSTAGES, WSTAGES>;
  static PerDeviceOnce attr;
  qg_status st = attr.run([&](int) {
    return check_cuda(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kTotal),
                      "cudaFuncSetAttribute(weight-only wide)");
  });
  if (st != QG_OK) return st;
  LaunchCfg lc((unsigned)(p.tiles_a * p.tiles_b * p.splits), kWideThreads, L::kTotal, s, (unsigned)p.splits);
  return check_cuda(cudaLaunchKernelEx(&lc.cfg, kern, tmX, tmW, tmS, tmZ, tmY, p), "weight-only wide launch");
}

// M > 64: BN = 128 token rows for M <= 128, else 256 (several token tiles above
// 256).  One CTA per SM; K is split across a cluster while the weight tiles
// alone leave SMs idle and every split keeps at least four K blocks.
qg_status launch_wonly_wide(bool w4, const void* x, int64_t ldx, const void* w, int64_t ldw_bytes,
                            const void* scale, const void* zero, const float* ws, const float* bias, void* y,
                            int64_t ldy, int64_t M, int64_t N, int64_t K, cudaStream_t s, int act, bool sym,
                            unsigned flags, int bn_force) {
  WideParams p = {};
  p.M = (int)M;
  p.N = (int)N;
  p.K = (int)K;
  p.nkb = (int)((K + kWideKB - 1) / kWideKB);
  p.w_scale = ws;
  p.bias = bias;
  p.y = static_cast<__half*>(y);
  p.ldy = ldy;
  p.act = act;
  p.sym = sym ? 1 : 0;
  p.static_w = (flags & QG_FLAG_STATIC_WEIGHTS) ? 1 : 0;
  const int bn = (bn_force == 128 || bn_force == 256) ? bn_force : (M <= 128 ? 128 : 256);
  p.tiles_a = (int)((N + 127) / 128);
  p.tiles_b = (int)((M + bn - 1) / bn);
  const int sms = sm_count();
  const int tiles = p.tiles_a * p.tiles_b;
  int splits = 1;
  const int max_splits = bn >= 256 ? 4 : 8;  // WideLayout::kMaxSplits
  while (splits < max_splits && tiles * splits * 2 <= sms && p.nkb >= 4 * splits * 2) splits *= 2;
  p.splits = splits;

  CUtensorMap tmX, tmW, tmS, tmZ;
  qg_status st;
  if ((st = make_tmap_2d(&tmX, x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, (uint64_t)K, (uint64_t)M, (uint64_t)ldx, 64,
                         (uint32_t)bn, CU_TENSOR_MAP_SWIZZLE_128B)) != QG_OK)
    return st;
  if (w4) {
    if ((st = make_tmap_2d(&tmW, w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)(K / 2), (uint64_t)N,
                           (uint64_t)ldw_bytes, 64, 128, CU_TENSOR_MAP_SWIZZLE_64B)) != QG_OK)
      return st;
    if ((st = make_tmap_2d(&tmS, scale, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, (uint64_t)N, (uint64_t)(K / 64),
                           (uint64_t)N, 128, 2, CU_TENSOR_MAP_SWIZZLE_NONE)) != QG_OK)
      return st;
    if (sym) {
      tmZ = tmS;  // never loaded
    } else if ((st = make_tmap_2d(&tmZ, zero, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, (uint64_t)N, (uint64_t)(K / 64),
                                  (uint64_t)N, 128, 2, CU_TENSOR_MAP_SWIZZLE_NONE)) != QG_OK) {
      return st;
    }
  } else {
    if ((st = make_tmap_2d(&tmW, w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)K, (uint64_t)N,
                           (uint64_t)ldw_bytes, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B)) != QG_OK)
      return st;
    tmS = tmW;
    tmZ = tmW;
  }
  // Without a K split, Y goes out by TMA stores of whole tiles (128 columns x
  // BN tokens) when its layout allows; the split-K tail stores from registers.
  CUtensorMap tmY = tmX;
  p.vec_y = (reinterpret_cast<uintptr_t>(y) % 16) == 0 && (ldy * 2) % 16 == 0;
  if (splits == 1 && p.vec_y) {
    if ((st = make_tmap_2d(&tmY, y, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, (uint64_t)N, (uint64_t)M, (uint64_t)ldy, 128,
                           (uint32_t)bn, CU_TENSOR_MAP_SWIZZLE_NONE)) != QG_OK)
      return st;
    p.tma_y = 1;
  }
  //                       BN   W4     XSTAGES WSTAGES
  if (bn == 128) return w4 ? run_wide<128, true, 10, 2>(tmX, tmW, tmS, tmZ, tmY, p, s)
                           : run_wide<128, false, 10, 2>(tmX, tmW, tmS, tmZ, tmY, p, s);
  return w4 ? run_wide<256, true, 6, 2>(tmX, tmW, tmS, tmZ, tmY, p, s)
            : run_wide<256, false, 6, 2>(tmX, tmW, tmS, tmZ, tmY, p, s);
}

}  // namespace qg

// qg_gemm_w8a8.cu -- W8A8 GEMM on the sm_100a tensor cores (tcgen05 kind::i8).
//
//   Y[m,n] = float(acc[m,n]) * (x_scale[m] * w_scale[n]) + bias[n]
//   acc[m,n] = sum_k Xq[m,k] * Wq[k,n]   (int8 x int8 -> int32, exact)
//
// Page "量化算法的本质", W8A8矩阵乘法 (Y = (x_scale*X)@(w_scale*W)+bias; the
// cuBLAS int32 buffer + second post-processing kernel is the slow variant this
// kernel replaces); page "量化与多精度算子" §四 (int32 accumulation, dequant in
// the epilogue while the result is on chip); page "Ascend C per-channel INT8
// GEMM" §5.3-5.4 (K tiles prefetched ahead of the MMA, scale at write-back).
//
// Structure (one CTA per SM, 6 warps):
//   warp 0      TMA producer: K-blocks of 128 bytes of both operands into a
//               ring of STAGES shared-memory stages (128-byte swizzle).
//   warp 1      allocates TMEM; one thread issues tcgen05.mma (M=128, N=BN,
//               K=32 per instruction, 4 per stage) and commits completion to
//               the stage's "empty" barrier and, per tile, to "tmem full".
//   warps 2..5  epilogue: tcgen05.ld the int32 accumulator, apply the scales
//               and bias in fp32, convert, store.  The accumulator is double
//               buffered in TMEM so the epilogue of tile i overlaps the
//               mainloop of tile i+1; int32 never reaches global memory.
// Operand roles: the "A" operand fills the 128 TMEM lanes (MMA M), "B" the
// columns (MMA N).  Prefill uses A = Xq, B = Wq.  Decode (small M) swaps them
// (A = Wq, B = Xq padded to 16..64 rows) and splits K across a thread-block
// cluster whose CTAs add their int32 partial tiles through distributed shared
// memory (exact in any order), so no partial sums go to global memory either.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "qg_dequant.cuh"
#include "qg_device.cuh"
#include "qg_internal.h"
#include "qg_quant_math.cuh"
#include "qg_w8a8_common.cuh"

namespace qg {

static __device__ unsigned long long g_status_w8a8;

unsigned long long read_clear_status_w8a8(cudaStream_t s) {
  unsigned long long v = 0, z = 0;
  cudaMemcpyFromSymbolAsync(&v, g_status_w8a8, sizeof(v), 0, cudaMemcpyDeviceToHost, s);
  cudaMemcpyToSymbolAsync(g_status_w8a8, &z, sizeof(z), 0, cudaMemcpyHostToDevice, s);
  cudaStreamSynchronize(s);
  return v;
}

// 6 warps; the fused quantize + decode kernel adds 4 quantizer warps, the
// int4-weight kernel 8 unpacking warps.
__host__ __device__ constexpr int w8a8_conv_warps(bool fuseq, bool w4) { return fuseq ? 4 : (w4 ? 8 : 0); }
__host__ __device__ constexpr int w8a8_threads(bool fuseq, bool w4 = false) {
  return 192 + 32 * w8a8_conv_warps(fuseq, w4);
}

template <int BN, int STAGES, bool SWAP, bool FUSEQ = false, bool W4 = false>
struct W8A8Smem {
  static constexpr int kA = 128 * kBK;                 // bytes per A stage
  static constexpr int kB = BN * kBK;                  // bytes per B stage
  // FUSEQ: the fp16 X tile of the stage; W4: the packed int4 weight tile (64 B rows)
  static constexpr int kX = FUSEQ ? BN * kBK * 2 : (W4 ? 128 * kBK / 2 : 0);
  static constexpr int kRing = STAGES * (kA + kB + kX);
  static constexpr int kRedLd = BN + 4;                // int32 row pitch of the split-K buffer
  static constexpr int kRed = SWAP ? 128 * kRedLd * 4 : 0;  // receives peers' partial rows
  static constexpr int kData = kRing + kRed;
  static constexpr int kBars = (3 * STAGES + 5) * 8 + 16;
  // staged w_scale/bias/w_zero/w_qsum (256 each); x_scale, 127/amax, partial
  // amax, x_zero, x_qsum (64 each)
  static constexpr int kEpi = 4 * 256 * 4 + 5 * 64 * 4;
  static constexpr int kTotal = 1024 + kData + kBars + kEpi;  // + alignment slack
  static constexpr int kAccBufs = SWAP ? 1 : 2;
  // FUSEQ / W4: converter warp groups taking alternate K blocks (must divide STAGES)
  static constexpr int kQGroups = STAGES % 4 == 0 ? 4 : 2;
  static constexpr int kConvWarps = w8a8_conv_warps(FUSEQ, W4);
  // converter warps per group (1 where there are none: keeps dead code well defined)
  static constexpr int kWpg = kConvWarps >= kQGroups ? kConvWarps / kQGroups : 1;
  static_assert(STAGES % kQGroups == 0, "each ring stage belongs to one quantizer group");
  // Narrow decode tiles: independent accumulators that successive MMAs rotate
  // through, so the tensor core pipelines them instead of serializing on one
  // accumulator (each N=16 MMA is a few cycles of math behind a long latency).
  static constexpr int kNAcc = SWAP ? (BN <= 16 ? 4 : (BN <= 32 ? 2 : 1)) : 1;
  // MMA issue of a narrow tile costs about the same per instruction whatever its
  // N, and that cost is per issuing thread: decode tiles spread each K block's
  // MMAs over kIssuers threads (one per accumulator), each in its own warp.
  static constexpr int kIssuers = kNAcc;
  static constexpr int kCols = kAccBufs * BN > kNAcc * BN ? kAccBufs * BN : kNAcc * BN;
  static constexpr int kTmemCols = kCols <= 32    ? 32
                                   : kCols <= 64  ? 64
                                   : kCols <= 128 ? 128
                                   : kCols <= 256 ? 256
                                                  : 512;
};

// 16 accumulator columns summed over the NACC rotating accumulators (int32,
// exact in any order).
template <int NACC, int BN>
__device__ __forceinline__ void load_acc16(uint32_t taddr, uint32_t (&r)[16]) {
  tmem_ld16(taddr, r);
  if (NACC > 1) {
    uint32_t t[NACC > 1 ? NACC - 1 : 1][16];
#pragma unroll
    for (int a = 1; a < NACC; ++a) tmem_ld16(taddr + (uint32_t)(a * BN), t[a - 1]);
    tmem_ld_wait();
#pragma unroll
    for (int a = 1; a < NACC; ++a)
#pragma unroll
      for (int j = 0; j < 16; ++j) r[j] = (uint32_t)((int32_t)r[j] + (int32_t)t[a - 1][j]);
  } else {
    tmem_ld_wait();
  }
}

template <int BN, int STAGES, bool SWAP, bool FUSEQ, bool ZP, bool W4>
__global__ void __launch_bounds__(w8a8_threads(FUSEQ, W4), 1)
    w8a8_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const W8A8Params p) {
  static_assert(!FUSEQ || SWAP, "the fused quantizer feeds the decode (swap-AB) kernel");
  static_assert(!(FUSEQ && ZP), "the fused quantizer is symmetric");
  static_assert(!W4 || (SWAP && !FUSEQ && !ZP), "int4 weights feed the swap-AB kernel as its A operand");
  using L = W8A8Smem<BN, STAGES, SWAP, FUSEQ, W4>;
  constexpr int kThreads = w8a8_threads(FUSEQ, W4);
  constexpr uint32_t kIdesc = idesc_i8_s32(128, BN);
  // with FUSEQ the B operand (Xq) is written by the quantizer warps, not by TMA
  // with W4 the A operand (int8 weights) is written by the unpacking warps
  constexpr uint32_t kStageBytes = (uint32_t)((W4 ? 0 : L::kA) + (FUSEQ ? 0 : L::kB));

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_base = smem_u32(smem_raw);
  const uint32_t base = (raw_base + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw_base);
  const uint32_t sA = base;
  const uint32_t sB = base + STAGES * L::kA;
  const uint32_t sX = base + STAGES * (L::kA + L::kB);  // FUSEQ: X tiles; W4: packed weights
  const uint32_t sRed = base + L::kRing;  // split-K receive buffer (its own region)
  const uint32_t bars = base + L::kData;
  auto full_bar = [&](int s) { return bars + 8u * s; };
  auto empty_bar = [&](int s) { return bars + 8u * (STAGES + s); };
  auto tfull_bar = [&](int b) { return bars + 8u * (2 * STAGES + b); };
  auto tempty_bar = [&](int b) { return bars + 8u * (2 * STAGES + 2 + b); };
  auto xfull_bar = [&](int s) { return bars + 8u * (2 * STAGES + 4 + s); };  // FUSEQ: X tile landed
  // split-K decode: every partial of the rows this CTA finishes has arrived
  const uint32_t red_full = bars + 8u * (3 * STAGES + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + L::kData + (3 * STAGES + 5) * 8);
  float* sWs = reinterpret_cast<float*>(gbase + L::kData + L::kBars);  // [256]
  float* sBias = sWs + 256;                                            // [256]
  float* sXs = sBias + 256;                                            // [64]
  float* sInv = sXs + 64;                                              // [64] FUSEQ: 127 / amax
  float* sPart = sInv + 64;                                            // [64] FUSEQ: amax over this CTA's K range
  float* sXz = sPart + 64;                                             // [64] ZP: x_zero
  int32_t* sXsum = reinterpret_cast<int32_t*>(sXz + 64);               // [64] ZP: x_qsum
  float* sWz = reinterpret_cast<float*>(sXsum + 64);                   // [256] ZP: w_zero
  int32_t* sWsum = reinterpret_cast<int32_t*>(sWz + 256);              // [256] ZP: w_qsum

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  unsigned long long* status = &g_status_w8a8;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1 + (L::kConvWarps > 0 ? L::kWpg : 0));  // TMA (+ one converter group)
      mbar_init(empty_bar(s), L::kIssuers);  // one commit per MMA-issuing thread
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull_bar(b), L::kIssuers);
      mbar_init(tempty_bar(b), 4);
    }
    if (FUSEQ || W4)
      for (int s = 0; s < STAGES; ++s) mbar_init(xfull_bar(s), 1);
    mbar_init(red_full, 1);
    if (SWAP && p.splits > 1)  // S CTAs x 128/S rows x BN int32, counted on arrival
      mbar_arrive_expect_tx(red_full, (uint32_t)(128 * BN * 4));
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), L::kTmemCols);
    tmem_relinquish();
  }
  // TMA issue of the weight part and the activation part of ring stage s for
  // K block kb of tile (ta, tb) (producer thread).
  const uint64_t pol_a = SWAP ? policy_evict_first() : policy_evict_last();
  const uint64_t pol_b = policy_evict_last();
  auto issue_w = [&](int s, int kb, int ta) {
    if (W4) {
      // packed int4 weight tile for the unpacking warps
      mbar_arrive_expect_tx(xfull_bar(s), (uint32_t)L::kX);
      if (tma_ok(sX + s * L::kX, kb * (kBK / 2), 1, status, 60))
        tma_load_2d_hint(sX + s * L::kX, &tmA, xfull_bar(s), kb * (kBK / 2), ta * 128, pol_a);
    } else {
      mbar_arrive_expect_tx(full_bar(s), kStageBytes);
      if (tma_ok(sA + s * L::kA, kb * kBK, 1, status, 61))
        tma_load_2d_hint(sA + s * L::kA, &tmA, full_bar(s), kb * kBK, ta * 128, pol_a);
    }
  };
  auto issue_x = [&](int s, int kb, int tb) {
    if (W4) mbar_arrive_expect_tx(full_bar(s), kStageBytes);
    if (!FUSEQ) {
      if (tma_ok(sB + s * L::kB, kb * kBK, 1, status, 62))
        tma_load_2d_hint(sB + s * L::kB, &tmB, full_bar(s), kb * kBK, tb * BN, pol_b);
    } else {
      // fp16 X tile for the quantizer warps (rows past M and K read as zero)
      mbar_arrive_expect_tx(xfull_bar(s), (uint32_t)L::kX);
      if (tma_ok(sX + s * L::kX, kb * kBK, 2, status, 63))
        tma_load_2d_hint(sX + s * L::kX, &tmB, xfull_bar(s), kb * kBK, tb * BN, pol_b);
    }
  };
  // Static weights (decode): the weight part of the first half of the ring of
  // this CTA's one work unit is issued now, before the wait on the preceding
  // kernel (which writes no weights, by the caller's contract).
  int npre = 0;
  if (SWAP && p.static_w && warp == 0 && lane == 0 && (int)blockIdx.x < p.tiles_a * p.tiles_b * p.splits) {
    const int split = (int)blockIdx.x % p.splits;
    int ta, tb;
    tile_coords((int)blockIdx.x / p.splits, p.tiles_a, p.tiles_b, ta, tb);
    const int kb0 = split * p.nkb / p.splits, kb1 = (split + 1) * p.nkb / p.splits;
    npre = min((STAGES + 1) / 2, kb1 - kb0);  // half the ring: more competes with the preceding kernel
    for (int i = 0; i < npre; ++i) issue_w(i, kb0 + i, ta);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const bool clustered = SWAP && p.splits > 1;
  // Split cluster barrier, matched by one cluster_wait() per thread before any
  // DSMEM access.  With FUSEQ the eight row-scale warps arrive later, after
  // publishing their partial row maxima (see row_scales).
  if (clustered && (!FUSEQ || warp < 2)) cluster_arrive_relaxed();
  pdl_trigger();
  pdl_wait();  // inputs of the preceding kernel are visible from here on

  const int num_tiles = p.tiles_a * p.tiles_b;
  const int units = num_tiles * p.splits;
  const bool scaled = p.out_dtype != QG_I32;
  bool ok = true;
  bool waited = false;  // this thread has done the cluster_wait() matching the early arrive

  // MMA issue loop of issuer `iss` (0..kIssuers-1): K steps k with
  // k % kIssuers == iss of every K block, into accumulator `iss`.
  auto issue_mma = [&](int iss) -> bool {
    int it = 0, tcount = 0;
    for (int u = blockIdx.x; u < units; u += gridDim.x, ++tcount) {
      const int split = u % p.splits;
      const int kb0 = split * p.nkb / p.splits, kb1 = (split + 1) * p.nkb / p.splits;
      const int buf = tcount % L::kAccBufs;
      const uint32_t tph = (uint32_t)(tcount / L::kAccBufs) & 1u;
      if (!mbar_wait(tempty_bar(buf), tph ^ 1u, status, 2)) return false;
      tc_fence_after();
      const uint32_t d = tmem + (uint32_t)(buf * BN + iss * BN);
      bool first = true;
      for (int kb = kb0; kb < kb1; ++kb, ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
        if (!mbar_wait(full_bar(s), ph, status, 3)) return false;
        tc_fence_after();
        const uint64_t da = sdesc_sw128(sA + s * L::kA);
        const uint64_t db = sdesc_sw128(sB + s * L::kB);
#pragma unroll
        for (int k = iss; k < kBK / 32; k += L::kIssuers) {
          mma_i8(d, da + 2u * k, db + 2u * k, kIdesc, first ? 0u : 1u);
          first = false;
        }
        mma_commit(empty_bar(s));
      }
      mma_commit(tfull_bar(buf));
    }
    return true;
  };

  // FUSEQ pass 1, run by warps 2..9 (the epilogue/MMA warps are idle until the
  // first B stage exists): per-row absmax of X, 16 loads in flight per lane,
  // then x_scale and 127/amax of each of the BN rows into shared memory.  Every
  // CTA needs the full-row scale; in a K-split cluster each CTA reads only its
  // own K range and the partial maxima are combined through distributed shared
  // memory (max is exact in any order).  Ends with a barrier of the eight warps,
  // after which sXs/sInv are visible to them.
  auto row_scales = [&](int ta, int tb, int split) {
    const int w8 = warp - 2;  // 0..7
    const int S = p.splits;
    const int v0 = S > 1 ? split * p.nkb / S * (kBK / 8) : 0;  // this CTA's 8-element chunks
    const int v1 = S > 1 ? min((split + 1) * p.nkb / S * (kBK / 8), p.K / 8) : p.K / 8;
    const bool tail = S == 1 || split == S - 1;  // owns the last K % 8 elements
    for (int r = w8; r < BN; r += 8) {
      const int m = tb * BN + r;
      float a = 0.0f;
      if (m < p.M) {
        const __half* row = p.x + (int64_t)m * p.ldx;
        const uint4* rowv = reinterpret_cast<const uint4*>(row);
        for (int i0 = v0; i0 < v1; i0 += 32 * 16) {
          uint4 v[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int i = i0 + 32 * j + lane;
            v[j] = i < v1 ? __ldg(rowv + i) : make_uint4(0, 0, 0, 0);
          }
#pragma unroll
          for (int j = 0; j < 16; ++j) a = absmax8(v[j], a);
        }
        if (tail)
          for (int k = (p.K / 8) * 8 + lane; k < p.K; k += 32) a = fmaxf(a, fabsf(__half2float(row[k])));
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
      if (lane == 0) sPart[r] = a;
    }
    if (S > 1) {
      __syncwarp();
      cluster_arrive_release();  // publish sPart
      cluster_wait();            // every CTA of the cluster has published
      waited = true;
    }
    for (int r = w8; r < BN; r += 8) {
      const int m = tb * BN + r;
      float a = sPart[r];
      if (S > 1) {
        // lane q fetches cluster rank q's partial maximum: one round trip
        if (lane < S) a = ld_dsmem_f32(mapa_shared(smem_u32(&sPart[r]), (uint32_t)lane));
#pragma unroll
        for (int o = 4; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
      }
      if (lane == 0) {
        const bool valid = m < p.M;
        sXs[r] = (valid && scaled) ? quant_scale(a) : 0.0f;
        sInv[r] = valid ? quant_inv(a) : 0.0f;
        if (valid && ta == 0 && split == 0 && p.xs_out) p.xs_out[m] = quant_scale(a);
      }
    }
    named_barrier(2, 256);
  };
  (void)row_scales;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      int it = 0;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        const int tile = u / p.splits, split = u % p.splits;
        int ta, tb;
        tile_coords(tile, p.tiles_a, p.tiles_b, ta, tb);
        const int kb0 = split * p.nkb / p.splits, kb1 = (split + 1) * p.nkb / p.splits;
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if (it >= npre) {  // (stages below npre: weights issued before the wait)
            if (!mbar_wait(empty_bar(s), ph ^ 1u, status, 1)) { ok = false; break; }
            issue_w(s, kb, ta);
          }
          issue_x(s, kb, tb);
        }
      }
      // Wait (bounded) until every load this thread issued has landed, so that
      // no copy into this CTA's shared memory outlives it, whether or not the
      // consumers got to them.  After a normal run each wait is one poll.
      for (int i = it - 1; i >= 0 && i >= it - STAGES; --i) {
        const uint32_t ph = (uint32_t)(i / STAGES) & 1u;
        if (FUSEQ || W4) mbar_wait(xfull_bar(i % STAGES), ph, status, 9);
        mbar_wait(full_bar(i % STAGES), ph, status, 9);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (one thread; prefill) ----------------
    if (!SWAP && lane == 0) ok = issue_mma(0);
  } else if (W4 && warp >= 6) {
    // ---------------- int4 unpacking warps ----------------
    // Each K block's packed tile (row = 64 bytes, 64-byte swizzle: 16-byte chunk
    // c at c ^ ((row >> 1) & 3)) becomes the int8 A stage (row = 128 bytes,
    // 128-byte swizzle, the layout TMA would write).  Nibble j of a 32-bit word
    // is k = 8p + j, a two's-complement code in [-8, 7].
    constexpr int kQG = L::kQGroups, kWpg = L::kWpg;
    const int cw = warp - 6;
    const int g = cw / kWpg;                 // group: K blocks kb0 + g, kb0 + g + kQG, ...
    const int gt = (cw % kWpg) * 32 + lane;  // thread within the group
    const int split = (int)blockIdx.x % p.splits;
    const int kb0 = split * p.nkb / p.splits, kb1 = (split + 1) * p.nkb / p.splits;
    int s = g;
    uint32_t ph = 0;
    for (int kb = kb0 + g; kb < kb1 && ok; kb += kQG) {
      if (!mbar_wait(xfull_bar(s), ph, status, 13)) { ok = false; break; }
      const uint8_t* pst = gbase + (sX - base) + s * L::kX;
      uint8_t* ast = gbase + (sA - base) + s * L::kA;
      for (int r = gt; r < 128; r += 32 * kWpg) {
        const uint8_t* prow = pst + r * 64;
        uint8_t* arow = ast + r * 128;
#pragma unroll
        for (int c = 0; c < 4; ++c) {  // 16-byte packed chunk = 32 k = two 16-byte int8 chunks
          const uint4 v = *reinterpret_cast<const uint4*>(prow + ((c ^ ((r >> 1) & 3)) << 4));
          const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
          uint32_t o[8];
#pragma unroll
          for (int i = 0; i < 4; ++i) s4x8_to_s8x8(wv[i], o[2 * i], o[2 * i + 1]);
          *reinterpret_cast<uint4*>(arow + (((2 * c) ^ (r & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
          *reinterpret_cast<uint4*>(arow + (((2 * c + 1) ^ (r & 7)) << 4)) = make_uint4(o[4], o[5], o[6], o[7]);
        }
      }
      fence_proxy_async_smem();  // generic-proxy writes -> tensor core reads
      __syncwarp();
      if (lane == 0) mbar_arrive(full_bar(s));
      if ((s += kQG) >= STAGES) { s -= STAGES; ph ^= 1u; }
    }
  } else if (FUSEQ && warp >= 6) {
    // ---------------- quantizer warps (fused quantize + decode) ----------------
    // After the row scales are staged (pass 1, below with the epilogue warps),
    // each K block's fp16 X tile (TMA) is quantized into the B stage in the
    // 128-byte swizzled layout a TMA load of Xq would have written.
    // quantizer groups take alternate K blocks (STAGES is a multiple of the
    // group count, so each ring stage is only ever handled by one group)
    constexpr int kQG = L::kQGroups, kWpg = 4 / kQG;
    const int qw = warp - 6;
    const int g = qw / kWpg;                            // group
    const int gt = (qw % kWpg) * 32 + lane;             // thread within the group
    int ta, tb;
    tile_coords(blockIdx.x / p.splits, p.tiles_a, p.tiles_b, ta, tb);
    const int split = (int)blockIdx.x % p.splits;
    const int kb0 = split * p.nkb / p.splits, kb1 = (split + 1) * p.nkb / p.splits;
    const bool writer = ta == 0 && p.xq_out != nullptr;  // this CTA also writes the codes out
    row_scales(ta, tb, split);
    int s = g;
    uint32_t ph = 0;
    for (int kb = kb0 + g; kb < kb1 && ok; kb += kQG) {
      // the X tile is loaded only once stage s is free, so its B part is free too
      if (!mbar_wait(xfull_bar(s), ph, status, 10)) { ok = false; break; }
      const uint8_t* xst = gbase + (sX - base) + s * L::kX;
      uint8_t* bst = gbase + (sB - base) + s * L::kB;
      for (int ch = gt; ch < BN * 8; ch += 32 * kWpg) {
        const int r = ch >> 3, c = ch & 7;  // row, 16-element chunk of the 128-element K block
        const float inv = sInv[r];
        const uint4* src = reinterpret_cast<const uint4*>(xst + r * (kBK * 2) + c * 32);
        const uint2 lo = quant8(src[0], inv), hi = quant8(src[1], inv);
        const uint4 q = make_uint4(lo.x, lo.y, hi.x, hi.y);
        *reinterpret_cast<uint4*>(bst + r * 128 + ((c ^ (r & 7)) << 4)) = q;
        const int m = tb * BN + r, k0 = kb * kBK + c * 16;
        if (writer && m < p.M && k0 < p.K) {
          int8_t* dst = p.xq_out + (int64_t)m * p.ldxq + k0;
          if (k0 + 16 <= p.K) {
            *reinterpret_cast<uint4*>(dst) = q;
          } else {
            const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
            for (int j = 0; j < 16; ++j)
              if (k0 + j < p.K) dst[j] = (int8_t)((w[j >> 2] >> (8 * (j & 3))) & 0xFF);
          }
        }
      }
      fence_proxy_async_smem();  // generic-proxy writes -> tensor core reads
      __syncwarp();
      if (lane == 0) mbar_arrive(full_bar(s));
      if ((s += kQG) >= STAGES) { s -= STAGES; ph ^= 1u; }
    }
  } else {
    // ---------------- epilogue warps ----------------
    const int et = threadIdx.x - 64;  // 0..127
    const int quad = warp & 3;        // TMEM lanes 32*quad .. 32*quad+31
    const int row = quad * 32 + lane;
    int tcount = 0;
    if (SWAP) {
      // One tile per CTA: stage this tile's x_scale columns while the mainloop runs.
      int ta, tb;
      tile_coords(blockIdx.x / p.splits, p.tiles_a, p.tiles_b, ta, tb);
      if (!FUSEQ && et < BN) {
        const int m = tb * BN + et;
        sXs[et] = (scaled && m < p.M) ? __ldg(p.x_scale + m) : 0.0f;
        if (ZP) {
          sXz[et] = (p.x_zero && m < p.M) ? __ldg(p.x_zero + m) : 0.0f;
          sXsum[et] = (p.x_qsum && m < p.M) ? __ldg(p.x_qsum + m) : 0;
        }
      }
      if (FUSEQ) row_scales(ta, tb, (int)blockIdx.x % p.splits);
      if (p.splits > 1) {
        // rows this CTA will own in the cluster reduction
        const int S = p.splits, rows = 128 / S, rank = (int)cluster_ctarank();
        if (et < rows) {
          const int n = ta * 128 + rank * rows + et;
          sWs[et] = (scaled && n < p.N) ? __ldg(p.w_scale + n) : 0.0f;
          sBias[et] = (p.bias && n < p.N) ? __ldg(p.bias + n) : 0.0f;
          if (ZP) {
            sWz[et] = (p.w_zero && n < p.N) ? __ldg(p.w_zero + n) : 0.0f;
            sWsum[et] = (p.w_qsum && n < p.N) ? __ldg(p.w_qsum + n) : 0;
          }
        }
      }
      named_barrier(1, 128);
      // decode tiles: the epilogue warps issue the MMAs of the mainloop
      const int iss = warp - 2;
      if (iss < L::kIssuers && lane == 0) ok = issue_mma(iss);
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;  // warp-uniform for the .aligned loads
    }
    for (int u = blockIdx.x; u < units && ok; u += gridDim.x, ++tcount) {
      const int tile = u / p.splits;
      int ta, tb;
      tile_coords(tile, p.tiles_a, p.tiles_b, ta, tb);
      const int buf = tcount % L::kAccBufs;
      const uint32_t tph = (uint32_t)(tcount / L::kAccBufs) & 1u;
      if (!mbar_wait(tfull_bar(buf), tph, status, 4)) { ok = false; break; }
      tc_fence_after();
      const uint32_t tbase = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(buf * BN);

      if (!SWAP) {
        // lane = output row m, columns = output columns n
        const int m = ta * 128 + row;
        const float xs = (m < p.M && scaled) ? __ldg(p.x_scale + m) : 0.0f;
        const float xz = (ZP && p.x_zero && m < p.M) ? __ldg(p.x_zero + m) : 0.0f;
        const int32_t xsum = (ZP && p.x_qsum && m < p.M) ? __ldg(p.x_qsum + m) : 0;
        dispatch_act(p.act, [&](auto gelu) {
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 16) {
          // column scales and bias: the same 16 addresses for the whole warp
          // (broadcast, L1-resident after the first tile row), issued before the
          // TMEM load so their latency overlaps it
          const int n0 = tb * BN + c0;
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
      } else if (p.splits == 1) {
        // lane = output column n (a W row), columns = output rows m
        const int n = ta * 128 + row;
        const bool nvalid = n < p.N;
        const float ws = (nvalid && scaled) ? __ldg(p.w_scale + n) : 0.0f;
        const float b = (nvalid && p.bias) ? __ldg(p.bias + n) : 0.0f;
        const float wz = (ZP && nvalid && p.w_zero) ? __ldg(p.w_zero + n) : 0.0f;
        const int32_t wsum = (ZP && nvalid && p.w_qsum) ? __ldg(p.w_qsum + n) : 0;
        dispatch_act(p.act, [&](auto gelu) {
#pragma unroll 1
          for (int c0 = 0; c0 < BN; c0 += 16) {
            uint32_t r[16];
            load_acc16<L::kNAcc, BN>(tbase + (uint32_t)c0, r);
            float v[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const float a = ZP ? zp_corrected((int32_t)r[j], sXz[c0 + j], sXsum[c0 + j], wz, wsum, p.K)
                                 : (float)(int32_t)r[j];
              v[j] = fmaf(a, sXs[c0 + j] * ws, b);
            }
            apply_act_c<decltype(gelu)::value>(v);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int m = tb * BN + c0 + j;
              if (nvalid && m < p.M) store_out(p.y, p.out_dtype, (int64_t)m * p.ldy + n, v[j], (int32_t)r[j]);
            }
          }
        });
      } else {
        // split-K: push this CTA's int32 partial rows into the shared memory of
        // the cluster CTA that owns them (slot = this CTA's rank).
        const int S = p.splits, rows = 128 / S;
        const int owner = row / rows, lr = row % rows;
        const uint32_t rank = cluster_ctarank();
        const uint32_t dst = mapa_shared(
            sRed + (uint32_t)((((int)rank * rows + lr) * L::kRedLd) * 4), (uint32_t)owner);
        const uint32_t rbar = mapa_shared(red_full, (uint32_t)owner);
        if (!waited) cluster_wait();  // every CTA of the cluster has started
        waited = true;
        // debug library: this row's BN int32 partials fit the owner's receive area
        // (warp-uniform: the loop's tensor-memory loads are .aligned)
        const bool push_ok =
            dcheck_warp(in_area((int64_t)(((int)rank * rows + lr) * L::kRedLd) * 4, BN * 4, L::kRed), status, 70);
#pragma unroll 1
        for (int c0 = 0; c0 < BN && push_ok; c0 += 16) {
          uint32_t r[16];
          load_acc16<L::kNAcc, BN>(tbase + (uint32_t)c0, r);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            st_async_v4(dst + (uint32_t)((c0 + 4 * j) * 4), r[4 * j], r[4 * j + 1], r[4 * j + 2],
                        r[4 * j + 3], rbar);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty_bar(buf));
    }
  }

  // Lanes 1..31 of the producer and MMA warps arrive here while lane 0 may
  // still be in its loop: reconverge before the warp-collective (.aligned)
  // cluster barrier and TMEM deallocation below.
  __syncwarp();

  if (clustered) {
    // Each CTA waits until every partial of the rows it owns has arrived (its
    // own barrier counts the st.async bytes; no cluster-wide barrier between
    // the pushes and the sums), then sums them in rank order from its own
    // shared memory.  The second cluster barrier phase, arrived at here and
    // waited on only before exit, keeps every CTA alive until all have issued
    // their pushes.
    if (!waited) cluster_wait();
    cluster_arrive_relaxed();
    if (!mbar_wait(red_full, 0, status, 8)) ok = false;
    const int S = p.splits, rows = 128 / S;
    const int rank = (int)cluster_ctarank();
    int ta, tb;
    tile_coords(blockIdx.x / S, p.tiles_a, p.tiles_b, ta, tb);
    const int32_t* red = reinterpret_cast<const int32_t*>(gbase + L::kRing);
    constexpr int chunks = BN / 4;
    // rows = 128 / S is a power of two: thread t takes row t % rows
    // (consecutive threads: consecutive n, so the stores coalesce) and the
    // 4-column chunks t / rows, t / rows + slots, ...; the S partial loads are
    // unrolled (predicated on S) so they are all in flight together
    const int lgr = 31 - __clz(rows);
    const int slots = kThreads >> lgr;
    const int lr = threadIdx.x & (rows - 1);
    // debug library: the S partial rows this thread reads lie in the receive area
    const bool red_ok = dcheck(in_area((int64_t)((S - 1) * rows + lr) * L::kRedLd * 4, BN * 4, L::kRed), status, 71);
    dispatch_act(p.act, [&](auto gelu) {
      if (!red_ok) return;
      for (int ch = threadIdx.x >> lgr; ch < chunks; ch += slots) {
        const int c = 4 * ch;
        int4 acc = make_int4(0, 0, 0, 0);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          if (q < S) {
            const int4 v = *reinterpret_cast<const int4*>(red + (q * rows + lr) * L::kRedLd + c);
            acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
          }
        }
        const int n = ta * 128 + rank * rows + lr;
        if (n < p.N) {
          const float ws = sWs[lr], b = sBias[lr];
          const int a4[4] = {acc.x, acc.y, acc.z, acc.w};
          float v[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float a = ZP ? zp_corrected(a4[j], sXz[c + j], sXsum[c + j], sWz[lr], sWsum[lr], p.K)
                               : (float)a4[j];
            v[j] = fmaf(a, sXs[c + j] * ws, b);
          }
          apply_act_c<decltype(gelu)::value>(v);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int m = tb * BN + c + j;
            if (m < p.M) store_out(p.y, p.out_dtype, (int64_t)m * p.ldy + n, v[j], a4[j]);
          }
        }
      }
    });
    cluster_wait();
  }

  tc_fence_before();
  cta_barrier_all();  // every thread of every role is done with TMEM and shared memory
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// K == 0: the empty sum, Y = bias (or 0).
// ---------------------------------------------------------------------------
__global__ void fill_bias_kernel(const float* bias, void* y, int dtype, int64_t ldy, int M, int N, int act) {
  pdl_trigger();
  pdl_wait();
  const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (i >= (int64_t)M * N) return;
  const int m = (int)(i / N), n = (int)(i % N);
  const float b = bias ? bias[n] : 0.0f;
  store_out(y, dtype, (int64_t)m * ldy + n, apply_act(b, act), 0);
}

qg_status launch_fill_bias(const float* bias, void* y, int dtype, int64_t ldy, int64_t M, int64_t N,
                           cudaStream_t s, int act) {
  const int64_t total = M * N;
  LaunchCfg lc((unsigned)((total + 255) / 256), 256, 0, s);
  return check_cuda(cudaLaunchKernelEx(&lc.cfg, fill_bias_kernel, bias, y, dtype, ldy, (int)M, (int)N, act),
                    "fill_bias launch");
}

// ---------------------------------------------------------------------------
// Host launch
// ---------------------------------------------------------------------------
template <int BN, int STAGES, bool SWAP, bool FUSEQ = false, bool ZP = false, bool W4 = false>
static qg_status run_w8a8(const CUtensorMap& tmA, const CUtensorMap& tmB, W8A8Params p,
                          int grid, cudaStream_t s) {
  using L = W8A8Smem<BN, STAGES, SWAP, FUSEQ, W4>;
  static_assert(L::kTotal <= 232448, "above the per-block shared memory limit");
  auto kern = w8a8_kernel<BN, STAGES, SWAP, FUSEQ, ZP, W4>;
  static PerDeviceOnce attr;
  qg_status st = attr.run([&](int) {
    return check_cuda(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kTotal),
                      "cudaFuncSetAttribute(w8a8)");
  });
  if (st != QG_OK) return st;
  LaunchCfg lc((unsigned)grid, w8a8_threads(FUSEQ, W4), L::kTotal, s, (unsigned)p.splits);
  return check_cuda(cudaLaunchKernelEx(&lc.cfg, kern, tmA, tmB, p), "w8a8 launch");
}

// Cluster size (K splits) of a decode launch: one CTA per SM (the operand ring
// takes most of shared memory), so the cluster grows while every CTA still
// gets an SM of its own.
static int decode_splits(int tiles_a, int nkb, int sms) {
  int splits = 1;
  const int forced = tuning(kTuneW8A8Splits);
  if (forced > 0) {
    splits = forced;
  } else {
    while (splits < 8 && tiles_a * splits * 2 <= sms && splits * 2 <= nkb) splits *= 2;
  }
  if (splits > nkb) splits = 1;
  return splits;
}

template <bool ZP>
static qg_status dispatch_w8a8(W8A8Params p, const int8_t* xq, int64_t ldx, const int8_t* wq, int64_t ldw,
                               int64_t M, int64_t N, int64_t K, cudaStream_t s);

qg_status launch_w8a8(const int8_t* xq, int64_t ldx, const int8_t* wq, int64_t ldw, const float* xs,
                      const float* ws, const float* bias, void* y, int dtype, int64_t ldy, int64_t M,
                      int64_t N, int64_t K, cudaStream_t s, int act, unsigned flags) {
  W8A8Params p = {};
  p.act = act;
  p.static_w = (flags & QG_FLAG_STATIC_WEIGHTS) ? 1 : 0;
  p.M = (int)M;
  p.N = (int)N;
  p.K = (int)K;
  p.nkb = (int)((K + kBK - 1) / kBK);
  p.x_scale = xs;
  p.w_scale = ws;
  p.bias = bias;
  p.y = y;
  p.ldy = ldy;
  p.out_dtype = dtype;
  return dispatch_w8a8<false>(p, xq, ldx, wq, ldw, M, N, K, s);
}

qg_status launch_w8a8_zp(const int8_t* xq, int64_t ldx, const int8_t* wq, int64_t ldw, const float* xs,
                         const float* xz, const int32_t* xsum, const float* ws, const float* wz,
                         const int32_t* wsum, const float* bias, void* y, int dtype, int64_t ldy,
                         int64_t M, int64_t N, int64_t K, cudaStream_t s) {
  W8A8Params p = {};
  p.M = (int)M;
  p.N = (int)N;
  p.K = (int)K;
  p.nkb = (int)((K + kBK - 1) / kBK);
  p.x_scale = xs;
  p.w_scale = ws;
  p.bias = bias;
  p.y = y;
  p.ldy = ldy;
  p.out_dtype = dtype;
  p.x_zero = xz;
  p.x_qsum = xsum;
  p.w_zero = wz;
  p.w_qsum = wsum;
  return dispatch_w8a8<true>(p, xq, ldx, wq, ldw, M, N, K, s);
}

template <bool ZP>
static qg_status dispatch_w8a8(W8A8Params p, const int8_t* xq, int64_t ldx, const int8_t* wq, int64_t ldw,
                               int64_t M, int64_t N, int64_t K, cudaStream_t s) {
  const int sms = sm_count();
  CUtensorMap tmA, tmB;
  qg_status st;

  if (M <= 64) {
    // Decode: A = Wq (N rows on the TMEM lanes), B = Xq padded to BN rows.
    const int bn = M <= 16 ? 16 : (M <= 32 ? 32 : 64);
    p.tiles_a = (int)((N + 127) / 128);
    p.tiles_b = 1;
    p.splits = decode_splits(p.tiles_a, p.nkb, sms);
    if ((st = make_tmap_2d(&tmA, wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)K, (uint64_t)N,
                           (uint64_t)ldw, kBK, 128, CU_TENSOR_MAP_SWIZZLE_128B)) != QG_OK)
      return st;
    if ((st = make_tmap_2d(&tmB, xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)K, (uint64_t)M,
                           (uint64_t)ldx, kBK, (uint32_t)bn, CU_TENSOR_MAP_SWIZZLE_128B)) != QG_OK)
      return st;
    const int grid = p.tiles_a * p.tiles_b * p.splits;
    if (bn == 16) return run_w8a8<16, 8, true, false, ZP>(tmA, tmB, p, grid, s);
    if (bn == 32) return run_w8a8<32, 8, true, false, ZP>(tmA, tmB, p, grid, s);
    return run_w8a8<64, 6, true, false, ZP>(tmA, tmB, p, grid, s);
  }

  // Prefill above 128 rows: 256 x 256 tiles on CTA pairs (half the shared-memory
  // operand traffic per SM of a one-SM tile).  The QG_W8A8_PAIR switch set to 0
  // keeps the one-SM tiles.
  if (M > 128 && tuning(kTuneW8A8Pair) != 0) return launch_w8a8_pair<ZP>(p, xq, ldx, wq, ldw, s);

  // Prefill: A = Xq (M rows), B = Wq (N rows), persistent over 128 x 256 tiles.
  constexpr int BN = 256;
  p.tiles_a = (int)((M + 127) / 128);
  p.tiles_b = (int)((N + BN - 1) / BN);
  p.splits = 1;
  if ((st = make_tmap_2d(&tmA, xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)K, (uint64_t)M,
                         (uint64_t)ldx, kBK, 128, CU_TENSOR_MAP_SWIZZLE_128B)) != QG_OK)
    return st;
  if ((st = make_tmap_2d(&tmB, wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)K, (uint64_t)N,
                         (uint64_t)ldw, kBK, BN, CU_TENSOR_MAP_SWIZZLE_128B)) != QG_OK)
    return st;
  const int tiles = p.tiles_a * p.tiles_b;
  const int grid = tiles < sms ? tiles : sms;
  return run_w8a8<BN, 4, false, false, ZP>(tmA, tmB, p, grid, s);
}

qg_status launch_w4a8(const int8_t* xq, int64_t ldx, const int32_t* qweight, const float* xs,
                      const float* ws, const float* bias, void* y, int dtype, int64_t ldy, int64_t M,
                      int64_t N, int64_t K, cudaStream_t s, int act) {
  // decode batches: the weight-only pipeline with an int8 A operand in tensor memory
  if (M <= 64 && act == QG_ACT_NONE)
    return launch_w4a8_decode(xq, ldx, qweight, xs, ws, bias, y, dtype, ldy, M, N, K, s);
  W8A8Params p = {};
  p.M = (int)M;
  p.N = (int)N;
  p.K = (int)K;
  p.nkb = (int)((K + kBK - 1) / kBK);
  p.x_scale = xs;
  p.w_scale = ws;
  p.bias = bias;
  p.y = y;
  p.ldy = ldy;
  p.out_dtype = dtype;
  p.act = act;
  // swap-AB for every M: the unpacked weight tile fills the 128 TMEM lanes;
  // larger batches take several 64-row tiles of Xq (no K split then)
  const int bn = M <= 16 ? 16 : (M <= 32 ? 32 : 64);
  p.tiles_a = (int)((N + 127) / 128);
  p.tiles_b = (int)((M + bn - 1) / bn);
  p.splits = p.tiles_b == 1 ? decode_splits(p.tiles_a, p.nkb, sm_count()) : 1;
  CUtensorMap tmA, tmB;
  qg_status st;
  if ((st = make_tmap_2d(&tmA, qweight, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)(K / 2), (uint64_t)N,
                         (uint64_t)(K / 2), kBK / 2, 128, CU_TENSOR_MAP_SWIZZLE_64B)) != QG_OK)
    return st;
  if ((st = make_tmap_2d(&tmB, xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)K, (uint64_t)M,
                         (uint64_t)ldx, kBK, (uint32_t)bn, CU_TENSOR_MAP_SWIZZLE_128B)) != QG_OK)
    return st;
  const int grid = p.tiles_a * p.tiles_b * p.splits;
  if (bn == 16) return run_w8a8<16, 8, true, false, false, true>(tmA, tmB, p, grid, s);
  if (bn == 32) return run_w8a8<32, 6, true, false, false, true>(tmA, tmB, p, grid, s);
  return run_w8a8<64, 4, true, false, false, true>(tmA, tmB, p, grid, s);
}

qg_status launch_quantize_w8a8(const void* x, int64_t ldx, const int8_t* wq, int64_t ldw,
                               const float* ws, const float* bias, void* y, int dtype, int64_t ldy,
                               int8_t* xq_out, int64_t ldxq, float* xs_out, int64_t M, int64_t N,
                               int64_t K, cudaStream_t s) {
  W8A8Params p = {};
  p.M = (int)M;
  p.N = (int)N;
  p.K = (int)K;
  p.nkb = (int)((K + kBK - 1) / kBK);
  p.w_scale = ws;
  p.bias = bias;
  p.y = y;
  p.ldy = ldy;
  p.out_dtype = dtype;
  p.x = static_cast<const __half*>(x);
  p.ldx = ldx;
  p.xq_out = xq_out;
  p.ldxq = ldxq;
  p.xs_out = xs_out;
  const int bn = M <= 16 ? 16 : (M <= 32 ? 32 : 64);
  p.tiles_a = (int)((N + 127) / 128);
  p.tiles_b = 1;
  p.splits = decode_splits(p.tiles_a, p.nkb, sm_count());
  CUtensorMap tmA, tmX;
  qg_status st = make_tmap_2d(&tmA, wq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)K, (uint64_t)N,
                              (uint64_t)ldw, kBK, 128, CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != QG_OK) return st;
  // fp16 X tiles of BN rows x 128 elements, unswizzled (row pitch 256 bytes)
  st = make_tmap_2d(&tmX, x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, (uint64_t)K, (uint64_t)M,
                    (uint64_t)ldx, kBK, (uint32_t)bn, CU_TENSOR_MAP_SWIZZLE_NONE);
  if (st != QG_OK) return st;
  const int grid = p.tiles_a * p.splits;
  if (bn == 16) return run_w8a8<16, 8, true, true>(tmA, tmX, p, grid, s);
  if (bn == 32) return run_w8a8<32, 6, true, true>(tmA, tmX, p, grid, s);
  return run_w8a8<64, 4, true, true>(tmA, tmX, p, grid, s);
}

}  // namespace qg

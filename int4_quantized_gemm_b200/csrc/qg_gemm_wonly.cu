// qg_gemm_wonly.cu -- weight-only GEMMs on the sm_100a tensor cores:
//
//   W8A16:  Y[m,n] = w_scale[n] * sum_k X[m,k] * Wq[k,n] + bias[n]
//   W4A16:  Y[m,n] = sum_k X[m,k] * (q[k,n] - z[k/64,n]) * s[k/64,n] + bias[n]
//
// Page "量化与多精度算子" §四 (weights stored as INT4/INT8 to save bandwidth,
// dequantized to FP16 inside the kernel, FP16 GEMM; memory-bound decode);
// page "INT4/FP16混合精度GEMM" §3.2/§4.2 (unpack (w >> 4i) & 0xF, (q - zp) *
// scale, FP16 matmul with FP32 accumulation, FP16 out); page "从零实现大语言
// 模型 INT8 量化" (block-wise dequant, one block of 64 per scale/zero).
//
// Operand roles (swap-AB): the weight tile supplies the 128 TMEM lanes (MMA
// M = 128 output columns n), X supplies the MMA N dimension (BN = 16..256
// token rows).  Dataflow per K block of 128:
//   warp 0      TMA: raw weight tile (int8, or packed int4 + fp16 scale/zero)
//               and the fp16 X tile into a shared-memory ring.
//   8 warps     dequantize in registers and write the fp16 A operand straight
//               into tensor memory (tcgen05.st): lane n holds row n of A, two
//               fp16 per 32-bit column.  Two groups of four warps (one per TMEM
//               lane quadrant) take alternate K blocks.
//   warps 1..4  one thread each issues tcgen05.mma kind::f16 with A from TMEM
//               and B = X from shared memory, fp32 accumulation in TMEM (one
//               to four issuers, see wonly_issuers).
// Keeping the dequantized weights out of shared memory keeps shared-memory
// traffic at about one byte per weight, far below what the tensor core needs
// to stay HBM-bound.  int8 codes and int4 (q - z) become fp16 exactly; W4A16
// rounds once, (q - z) * s, to fp16.  K is split across a thread-block cluster
// whose CTAs add their fp32 partial tiles through distributed shared memory.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "qg_dequant.cuh"
#include "qg_device.cuh"
#include "qg_internal.h"

namespace qg {

static __device__ unsigned long long g_status_wonly;

unsigned long long read_clear_status_wonly(cudaStream_t s) {
  unsigned long long v = 0, z = 0;
  cudaMemcpyFromSymbolAsync(&v, g_status_wonly, sizeof(v), 0, cudaMemcpyDeviceToHost, s);
  cudaMemcpyToSymbolAsync(g_status_wonly, &z, sizeof(z), 0, cudaMemcpyHostToDevice, s);
  cudaStreamSynchronize(s);
  return v;
}

constexpr int kKB = 128;  // K elements per block
constexpr int kConvWarps = 8;
// Warps: 0 TMA producer; 1..kIssuers MMA issuers (warp 1 also owns TMEM);
// then 8 converter warps.  A narrow (N = 16, 32) MMA costs about the same issue
// time per instruction as a wide one and that cost is per issuing thread, so
// narrow tiles spread each K block's 8 MMAs over several issuing warps, each
// accumulating into its own TMEM tile.
__host__ __device__ constexpr int wonly_issuers(int bn) { return bn <= 16 ? 4 : (bn <= 32 ? 2 : 1); }
__host__ __device__ constexpr int wonly_threads(int bn) { return 32 * (1 + wonly_issuers(bn) + kConvWarps); }

struct WOnlyParams {
  int M, N, K;
  int tiles_a, tiles_b, nkb, splits;
  const float* w_scale;  // W8A16 only
  const float* bias;
  __half* y;
  int64_t ldy;
  int act;  // qg_activation applied to the fp32 value before the fp16 conversion
  int sym;  // W4: two's-complement codes, no zero points (z = 8 on the offset codes)
  // Fault injection for tests (qg_debug_inject_timeout), zero in every other
  // launch: withhold (1) the copy of CTA 0's first K block, and bound every
  // wait by dbg_wait_us microseconds instead of kWaitLimitNs (0).
  int dbg_withhold;
  uint32_t dbg_wait_us;
  // The caller guarantees that no kernel still in flight writes the weights
  // (codes, scales, zero points): the first ring stages of weights are then
  // loaded, and converted, before the wait on the preceding kernel.
  int static_w;
  // W4A8 (I8 kernels): int8 X codes with one fp32 scale per row, symmetric
  // int4 weights with one fp32 scale per column (w_scale), the W8A8 epilogue
  // and any output type (QG_I32: the raw int32 sums; the scales may be NULL)
  const float* x_scale;
  void* y_any;
  int out_dtype;
};

// I8: W4A8 on the int8 tensor path -- X is int8 (one 128-byte atom per row and
// K block), the int4 weights are unpacked to int8 (no scale/zero tiles), an A
// stage is 32 TMEM columns (four int8 per column) and the sums are int32.
template <int BN, bool W4, int STAGES, int ASTAGES, bool SPLITK, bool I8 = false>
struct WOnlyLayout {
  static constexpr int kX = I8 ? BN * 128 : BN * 256;      // fp16: two 128-byte-swizzled atoms of 64 K
  static constexpr int kW = W4 ? 128 * 64 : 128 * 128;     // packed int4 (64B rows) or int8 rows
  static constexpr int kSZ = (W4 && !I8) ? 2 * 128 * 2 : 0;  // scale tile [2 groups][128] fp16 (zero alike)
  static constexpr int kACols = I8 ? 32 : 64;              // tensor-memory columns of an A stage (128 K)
  static constexpr int kStage = kX + kW + 2 * kSZ;         // multiple of 1024
  static constexpr int kRing = STAGES * kStage;
  static constexpr int kRedLd = BN + 4;
  static constexpr int kRed = SPLITK ? (128 + 8) * kRedLd * 4 : 0;  // peers' fp32 partial rows
  static constexpr int kData = kRing + kRed;
  static constexpr int kBars = (3 * STAGES + 2 * ASTAGES + 2) * 8 + 16;
  static constexpr int kWTx = kW + 2 * kSZ;  // weight bytes of a stage (codes + scale + zero)
  static constexpr int kXTx = kX;            // activation bytes of a stage
  static constexpr int kEpi = 2 * 128 * 4;                 // staged w_scale / bias of owned rows
  static constexpr int kTotal = 1024 + kData + kBars + kEpi;
  static constexpr int kDCols = BN < 64 ? 64 : BN;         // accumulator columns
  // one accumulator per MMA-issuing warp, together filling kDCols
  static constexpr int kNAcc = kDCols / BN;
  static_assert(kNAcc == wonly_issuers(BN), "one accumulator per issuer");
  static constexpr int kNeed = kDCols + kACols * ASTAGES;  // + the A stages
  static constexpr int kTmemCols = kNeed <= 128 ? 128 : (kNeed <= 256 ? 256 : 512);
  static_assert(kStage % 1024 == 0, "stage must keep 1024-byte alignment");
  // The converter groups take alternate K blocks; with an even ring every
  // stage is only ever converted by one group, so a group's parity waits on it
  // are never more than one phase ahead of the barrier.
  static_assert(STAGES % 2 == 0, "the shared-memory ring must have an even number of stages");
  static_assert(kNeed <= 512, "tensor memory overflow");
};

// 8 accumulator columns summed over the NACC rotating accumulators, in
// accumulator order: fp32, or int32 (exact) for the int8 tensor path.
template <int NACC, int BN, bool INT = false>
__device__ __forceinline__ void load_acc8(uint32_t taddr, uint32_t (&v)[8]) {
  tmem_ld8(taddr, v);
  if (NACC > 1) {
    uint32_t t[NACC > 1 ? NACC - 1 : 1][8];
#pragma unroll
    for (int a = 1; a < NACC; ++a) tmem_ld8(taddr + (uint32_t)(a * BN), t[a - 1]);
    tmem_ld_wait();
#pragma unroll
    for (int a = 1; a < NACC; ++a)
#pragma unroll
      for (int j = 0; j < 8; ++j)
        v[j] = INT ? (uint32_t)((int32_t)v[j] + (int32_t)t[a - 1][j])
                   : __float_as_uint(__uint_as_float(v[j]) + __uint_as_float(t[a - 1][j]));
  } else {
    tmem_ld_wait();
  }
}

// One output of the W4A8 epilogue, as the W8A8 kernels form it:
// fmaf(float(acc), x_scale * w_scale, bias) in the output type, or the raw sum.
__device__ __forceinline__ void store_i8_out(void* y, int dtype, int64_t idx, int32_t acc, float xs, float ws,
                                             float b) {
  const float v = fmaf((float)acc, xs * ws, b);
  switch (dtype) {
    case QG_F32: static_cast<float*>(y)[idx] = v; break;
    case QG_F16: static_cast<__half*>(y)[idx] = __float2half_rn(v); break;
    case QG_BF16: static_cast<__nv_bfloat16*>(y)[idx] = __float2bfloat16_rn(v); break;
    default: static_cast<int32_t*>(y)[idx] = acc; break;
  }
}

template <int BN, bool W4, int STAGES, int ASTAGES, int MINB, bool SPLITK, bool I8 = false>
__global__ void __launch_bounds__(wonly_threads(BN), MINB)
    wonly_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                 const __grid_constant__ CUtensorMap tmS, const __grid_constant__ CUtensorMap tmZ,
                 const WOnlyParams p) {
  static_assert(!I8 || W4, "the int8 tensor path takes int4 weights (W4A8)");
  using L = WOnlyLayout<BN, W4, STAGES, ASTAGES, SPLITK, I8>;
  constexpr uint32_t kIdesc = I8 ? idesc_i8_s32(128, BN) : idesc_f16_f32(128, BN);
  constexpr int kMmas = I8 ? 4 : 8;  // MMAs per K block of 128 (K = 32 int8 or 16 fp16 each)
  constexpr int kIssuers = wonly_issuers(BN);
  constexpr int kThreadsW = wonly_threads(BN);
  constexpr int kConv0 = 1 + kIssuers;  // first converter warp

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_base = smem_u32(smem_raw);
  const uint32_t base = (raw_base + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw_base);
  const uint32_t bars = base + L::kData;
  auto w_full = [&](int s) { return bars + 8u * s; };               // weight part of stage s landed
  auto raw_empty = [&](int s) { return bars + 8u * (STAGES + s); };  // stage s consumed
  auto a_full = [&](int a) { return bars + 8u * (2 * STAGES + a); };
  auto a_empty = [&](int a) { return bars + 8u * (2 * STAGES + ASTAGES + a); };
  const uint32_t d_full = bars + 8u * (2 * STAGES + 2 * ASTAGES);
  auto x_full = [&](int s) { return bars + 8u * (2 * STAGES + 2 * ASTAGES + 1 + s); };  // X part landed
  // split-K: the partial rows this CTA finishes have all arrived (st.async bytes)
  const uint32_t red_full = bars + 8u * (3 * STAGES + 2 * ASTAGES + 1);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + L::kData + (3 * STAGES + 2 * ASTAGES + 2) * 8);
  float* sWs = reinterpret_cast<float*>(gbase + L::kData + L::kBars);  // [128]
  float* sBias = sWs + 128;                                            // [128]
  const uint32_t sRed = base + L::kRing;
  auto stage_x = [&](int s) { return base + (uint32_t)(s * L::kStage); };
  auto stage_w = [&](int s) { return base + (uint32_t)(s * L::kStage + L::kX); };
  auto stage_sc = [&](int s) { return base + (uint32_t)(s * L::kStage + L::kX + L::kW); };
  auto stage_ze = [&](int s) { return base + (uint32_t)(s * L::kStage + L::kX + L::kW + L::kSZ); };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  unsigned long long* status = &g_status_wonly;
  const uint64_t lim = p.dbg_wait_us ? (uint64_t)p.dbg_wait_us * 1000ull : kWaitLimitNs;

  // one work unit per CTA: (tile, split)
  const int S = SPLITK ? p.splits : 1;
  const int tile = blockIdx.x / S;
  const int split = blockIdx.x % S;
  const int ta = tile % p.tiles_a;  // weight rows (output columns n)
  const int tb = tile / p.tiles_a;  // X rows (tokens m)
  const int kb0 = split * p.nkb / S, kb1 = (split + 1) * p.nkb / S;

  // TMA issue of the two parts of ring stage s for K block kb (producer thread)
  const uint64_t pol_w = policy_evict_first();
  const uint64_t pol_x = policy_evict_last();
  auto load_w = [&](int s, int kb) {
    mbar_arrive_expect_tx(w_full(s), (uint32_t)(L::kWTx - (p.sym ? L::kSZ : 0)));
    if (W4) {
      if (tma_ok(stage_w(s), kb * (kKB / 2), 1, status, 60))
        tma_load_2d_hint(stage_w(s), &tmW, w_full(s), kb * (kKB / 2), ta * 128, pol_w);
      if (!I8 && tma_ok(stage_sc(s), ta * 128, 2, status, 61))
        tma_load_2d_hint(stage_sc(s), &tmS, w_full(s), ta * 128, kb * 2, pol_w);
      if (!I8 && !p.sym && tma_ok(stage_ze(s), ta * 128, 2, status, 62))
        tma_load_2d_hint(stage_ze(s), &tmZ, w_full(s), ta * 128, kb * 2, pol_w);
    } else {
      if (tma_ok(stage_w(s), kb * kKB, 1, status, 63))
        tma_load_2d_hint(stage_w(s), &tmW, w_full(s), kb * kKB, ta * 128, pol_w);
    }
  };
  auto load_x = [&](int s, int kb) {
    mbar_arrive_expect_tx(x_full(s), (uint32_t)L::kXTx);
    if (I8) {  // int8 codes: the block is one 128-byte atom per row
      if (tma_ok(stage_x(s), kb * kKB, 1, status, 64))
        tma_load_2d_hint(stage_x(s), &tmX, x_full(s), kb * kKB, tb * BN, pol_x);
      return;
    }
    if (tma_ok(stage_x(s), kb * kKB, 2, status, 64))
      tma_load_2d_hint(stage_x(s), &tmX, x_full(s), kb * kKB, tb * BN, pol_x);
    if (tma_ok(stage_x(s) + BN * 128, kb * kKB + 64, 2, status, 65))
      tma_load_2d_hint(stage_x(s) + BN * 128, &tmX, x_full(s), kb * kKB + 64, tb * BN, pol_x);
  };
  int npre = 0;  // ring stages whose weight part was issued before the wait

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(w_full(s), 1);
      mbar_init(x_full(s), 1);
      mbar_init(raw_empty(s), kConvWarps / 2 + kIssuers);  // one converter group (W) + MMA commits (X)
    }
    for (int a = 0; a < ASTAGES; ++a) {
      mbar_init(a_full(a), kConvWarps / 2);
      mbar_init(a_empty(a), kIssuers);
    }
    mbar_init(d_full, kIssuers);
    mbar_init(red_full, 1);
    fence_mbar_init();
    if (S > 1) {
      // every CTA of the cluster (itself included) sends its partial of each row
      // this CTA finishes: S x rows x BN fp32, counted on arrival
      const int rank = (int)cluster_ctarank();
      const int rows = (rank + 1) * 128 / S - rank * 128 / S;
      mbar_arrive_expect_tx(red_full, (uint32_t)(S * rows * BN * 4));
    }
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmW);
    if (W4 && !I8) {
      tma_prefetch_desc(&tmS);
      tma_prefetch_desc(&tmZ);
    }
    if (p.static_w) {
      // Static weights: the weight part of the first half of the ring goes
      // straight to shared memory now, before the wait on the preceding kernel
      // (which writes no weights, by the caller's contract), and the converters
      // turn it into A operands while that kernel finishes.  (A whole ring
      // measured slower: its loads compete with the preceding kernel's.)
      npre = min((STAGES + 1) / 2, kb1 - kb0);  // half the ring: more competes with the preceding kernel
      for (int i = 0; i < npre; ++i) {
        if (p.dbg_withhold && blockIdx.x == 0 && i == 0) continue;  // test-only: never lands
        load_w(i, kb0 + i);
      }
    }
    if (SPLITK) {
      // Decode: start the next half-ring of this CTA's weight blocks towards
      // L2 now, before the wait on the preceding kernel, so the ring's first
      // loads after the wait hit L2 instead of paying an HBM round trip.  More
      // than that competes with the preceding kernel's own weight stream.
      const int kend = min(kb1, kb0 + npre + (STAGES + 1) / 2);
      for (int kb = kb0 + npre; kb < kend; ++kb) {
        if (W4) {
          if (tma_ok(0u, kb * (kKB / 2), 1, status, 66)) tma_prefetch_l2_2d(&tmW, kb * (kKB / 2), ta * 128);
          if (!I8 && tma_ok(0u, ta * 128, 2, status, 67)) tma_prefetch_l2_2d(&tmS, ta * 128, kb * 2);
          if (!I8 && !p.sym && tma_ok(0u, ta * 128, 2, status, 68)) tma_prefetch_l2_2d(&tmZ, ta * 128, kb * 2);
        } else {
          if (tma_ok(0u, kb * kKB, 1, status, 69)) tma_prefetch_l2_2d(&tmW, kb * kKB, ta * 128);
        }
      }
    }
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (S > 1) cluster_arrive_relaxed();  // matched by cluster_wait() before any DSMEM access
  pdl_trigger();
  // Inputs of the preceding kernel are visible after the wait.  With static
  // weights the converter warps skip it: they read only weights, which no
  // kernel in flight writes (the flag's contract); X reaches the MMAs through
  // the producer, which waits, and the epilogue's stores follow those MMAs.
  // So the converters turn the prefetched stages into A operands while the
  // preceding kernel finishes.
  if (!p.static_w || warp < kConv0) pdl_wait();

  // rows [row_lo(r), row_lo(r+1)) of the tile are reduced by cluster rank r
  auto row_lo = [&](int r) { return r * 128 / S; };
  const int maxrows = (128 + S - 1) / S;
  bool ok = true;
  bool waited = false;  // this thread has done the cluster_wait() matching the early arrive

  if (warp == 0) {
    if (lane == 0) {
      int it = 0;
      for (int kb = kb0; kb < kb1; ++kb, ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
        if (it >= npre) {
          if (!mbar_wait(raw_empty(s), ph ^ 1u, status, 11, lim)) { ok = false; break; }
          if (p.dbg_withhold && blockIdx.x == 0 && it == 0) continue;  // test-only: this stage never lands
          load_w(s, kb);
        } else if (p.dbg_withhold && blockIdx.x == 0 && it == 0) {
          continue;
        }
        load_x(s, kb);
      }
      // Wait (bounded) until every load this thread issued has landed, so that
      // no copy into this CTA's shared memory outlives it, whether or not the
      // consumers got to them (they may have given up).  After a normal run
      // these phases are complete and each wait is one poll.
      for (int i = it - 1; i >= 0 && i >= it - STAGES; --i) {
        if (p.dbg_withhold && blockIdx.x == 0 && i == 0) continue;  // never issued
        mbar_wait(w_full(i % STAGES), (uint32_t)(i / STAGES) & 1u, status, 19, lim);
        mbar_wait(x_full(i % STAGES), (uint32_t)(i / STAGES) & 1u, status, 19, lim);
      }
    }
  } else if (warp < kConv0) {
    // ---------------- MMA issuers: issuer i takes K steps j % kIssuers == i ----------------
    const int iss = warp - 1;
    if (lane == 0) {
      int it = 0;
      const uint32_t d = tmem + (uint32_t)(iss * BN);
      for (int kb = kb0; kb < kb1; ++kb, ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
        const int a = it % ASTAGES;
        const uint32_t aph = (uint32_t)(it / ASTAGES) & 1u;
        if (!mbar_wait(x_full(s), ph, status, 12, lim)) { ok = false; break; }
        if (!mbar_wait(a_full(a), aph, status, 13, lim)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a_col = tmem + (uint32_t)(L::kDCols + L::kACols * a);
        // MMA j takes 32 bytes of K (16 fp16 or 32 int8): 8 A columns, and the
        // next 32 bytes of the 128-byte swizzled X rows (fp16: a second atom of
        // BN rows after the first 64 K)
#pragma unroll
        for (int j = iss; j < kMmas; j += kIssuers) {
          const uint64_t db = sdesc_sw128(stage_x(s) + (uint32_t)((j >> 2) * BN * 128 + (j & 3) * 32));
          if constexpr (I8) {
            mma_i8_ts(d, a_col + 8u * j, db, kIdesc, (kb > kb0 || j > iss) ? 1u : 0u);
          } else {
            mma_f16_ts(d, a_col + 8u * j, db, kIdesc, (kb > kb0 || j > iss) ? 1u : 0u);
          }
        }
        mma_commit(a_empty(a));
        mma_commit(raw_empty(s));
      }
      if (ok) mma_commit(d_full);
    }
  } else {
    // ---------------- converters, then epilogue ----------------
    const int quad = warp & 3;                // TMEM lane quadrant this warp may access
    const int grp = (warp - kConv0) >> 2;     // converter group (alternate K blocks)
    const int half = grp;                     // epilogue: which half of the accumulator columns
    const int row = quad * 32 + lane;         // TMEM lane = weight row within the tile
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    const int ct = threadIdx.x - 32 * kConv0;  // 0..255
    const int gt = ct & 127;                   // thread index within the converter group
    // epilogue constants, fetched while the mainloop runs
    const int n = ta * 128 + row;
    const bool nvalid = n < p.N;
    // column scale: W8A16's, or W4A8's (NULL for raw int32 output); W4A16 has none
    auto col_scale = [&](int nn) -> float {
      if (nn >= p.N) return 1.0f;
      if (I8) return p.w_scale ? __ldg(p.w_scale + nn) : 0.0f;
      return W4 ? 1.0f : __ldg(p.w_scale + nn);
    };
    const float my_ws = col_scale(n);
    const float my_b = (nvalid && p.bias) ? __ldg(p.bias + n) : 0.0f;
    if (S > 1 && ct < 128) {
      const int rank = (int)cluster_ctarank();
      const int rows = row_lo(rank + 1) - row_lo(rank);
      if (ct < rows) {
        const int nn = ta * 128 + row_lo(rank) + ct;
        sWs[ct] = col_scale(nn);
        sBias[ct] = (p.bias && nn < p.N) ? __ldg(p.bias + nn) : 0.0f;
      }
    }
    // The two converter groups take alternate K blocks (group g: blocks kb0 + g,
    // kb0 + g + 2, ...), each warp a whole block for its 32 rows, so the fixed
    // cost of a stage (waits, fences, arrivals) is paid once per 128 K.
    int it = grp;
    int s = grp, a = grp;
    uint32_t ph = 0, aph = 0;
    for (int kb = kb0 + grp; kb < kb1 && ok; kb += 2, it += 2) {
      if (!mbar_wait(w_full(s), ph, status, 14, lim)) { ok = false; break; }
      if (!mbar_wait(a_empty(a), aph ^ 1u, status, 15, lim)) { ok = false; break; }
      tc_fence_after();
      const uint32_t dst = tmem + lane_addr + (uint32_t)(L::kDCols + L::kACols * a);
      if constexpr (I8) {
        // W4A8: packed row of 64 bytes (64-byte swizzle: 16-byte chunk c, codes
        // k = 32c..32c+31, at c ^ ((row >> 1) & 3)) -> int8 codes in k order,
        // four per tensor-memory column; X stays as loaded
        const uint8_t* wrow = gbase + (stage_w(s) - base) + row * 64;
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2) {
          uint32_t r[16];
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            const int chunk = 2 * c2 + cc;
            const uint4 v = *reinterpret_cast<const uint4*>(wrow + ((chunk ^ ((row >> 1) & 3)) << 4));
            const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) s4x8_to_s8x8(wv[i], r[8 * cc + 2 * i], r[8 * cc + 2 * i + 1]);
          }
          tmem_st16(dst + 16 * c2, r);
        }
      } else if (W4) {
        // packed row: 64 bytes, 64-byte swizzle (16-byte chunk c at c ^ ((row >> 1) & 3));
        // chunks 0-1 belong to quantization group 0 of the block, 2-3 to group 1
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
            for (int i = 0; i < 4; ++i) u4x8_to_h2x4(wv[i], s2, c_lo, c_hi, m_lo, m_hi, r + 4 * i);
            tmem_st16(dst + 16 * chunk, r);
          }
        }
        // X of this stage into the (k, k+4) pair order (each 16-byte chunk in place;
        // the 128-byte swizzle moves whole chunks, so it is unaffected).  X may land
        // after the weights (static weights: only after the preceding kernel).
        if (!mbar_wait(x_full(s), ph, status, 17, lim)) {
          ok = false;
          tmem_st_wait();
          break;
        }
        uint8_t* xst = gbase + (stage_x(s) - base);
#pragma unroll
        for (int c = gt; c < BN * 16; c += 32 * kConvWarps / 2) permute_x_chunk(xst + 16 * c);
        fence_proxy_async_smem();  // generic-proxy writes -> tensor core reads
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
        mbar_arrive(raw_empty(s));
      }
      if ((s += 2) >= STAGES) { s -= STAGES; ph ^= 1u; }
      if ((a += 2) >= ASTAGES) { a -= ASTAGES; aph ^= 1u; }
    }
    (void)it;

    // epilogue: lane = output column n, accumulator columns = token rows m
    if (ok && mbar_wait(d_full, 0, status, 16, lim)) {
      tc_fence_after();
      constexpr int kHalfCols = BN / 2;
      if (S == 1) {
        if constexpr (I8) {
#pragma unroll 1
          for (int c0 = half * kHalfCols; c0 < (half + 1) * kHalfCols; c0 += 8) {
            uint32_t v[8];
            load_acc8<L::kNAcc, BN, true>(tmem + lane_addr + (uint32_t)c0, v);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const int m = tb * BN + c0 + j;
              if (nvalid && m < p.M)
                store_i8_out(p.y_any, p.out_dtype, (int64_t)m * p.ldy + n, (int32_t)v[j],
                             p.x_scale ? __ldg(p.x_scale + m) : 0.0f, my_ws, my_b);
            }
          }
        } else
        dispatch_act(p.act, [&](auto gelu) {
#pragma unroll 1
          for (int c0 = half * kHalfCols; c0 < (half + 1) * kHalfCols; c0 += 8) {
            uint32_t v[8];
            load_acc8<L::kNAcc, BN>(tmem + lane_addr + (uint32_t)c0, v);
            float f[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) f[j] = fmaf(__uint_as_float(v[j]), my_ws, my_b);
            apply_act_c<decltype(gelu)::value>(f);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const int m = tb * BN + c0 + j;
              if (nvalid && m < p.M) p.y[(int64_t)m * p.ldy + n] = __float2half_rn(f[j]);
            }
          }
        });
      } else {
        // push this CTA's fp32 partial row into the CTA that owns it (slot = rank)
        int owner = 0;
        while (owner + 1 < S && row >= row_lo(owner + 1)) ++owner;
        const int lr = row - row_lo(owner);
        const uint32_t rank = cluster_ctarank();
        const uint32_t dst = mapa_shared(
            sRed + (uint32_t)((((int)rank * maxrows + lr) * L::kRedLd) * 4), (uint32_t)owner);
        const uint32_t rbar = mapa_shared(red_full, (uint32_t)owner);
        cluster_wait();  // every CTA of the cluster has started
        waited = true;
        // debug library: this half row of fp32 partials fits the owner's receive area
        // (warp-uniform: the loop's tensor-memory loads are .aligned)
        const bool push_ok = dcheck_warp(
            in_area((int64_t)(((int)rank * maxrows + lr) * L::kRedLd + half * kHalfCols) * 4, kHalfCols * 4, L::kRed),
            status, 70);
#pragma unroll 1
        for (int c0 = half * kHalfCols; c0 < (half + 1) * kHalfCols && push_ok; c0 += 8) {
          uint32_t v[8];
          load_acc8<L::kNAcc, BN, I8>(tmem + lane_addr + (uint32_t)c0, v);
          st_async_v4(dst + (uint32_t)(c0 * 4), v[0], v[1], v[2], v[3], rbar);
          st_async_v4(dst + (uint32_t)(c0 * 4 + 16), v[4], v[5], v[6], v[7], rbar);
        }
      }
    } else {
      ok = false;
    }
  }

  __syncwarp();
  if (S > 1) {
    // Each CTA waits until every partial of the rows it finishes has arrived
    // (its own barrier counts the st.async bytes, so no cluster-wide barrier
    // sits between the pushes and the sums), then sums them in rank order
    // (deterministic).  A second cluster barrier phase, arrived at here and
    // waited on only before exit, keeps every CTA alive until all have issued
    // their pushes.
    if (!waited) cluster_wait();
    cluster_arrive_relaxed();
    if (!mbar_wait(red_full, 0, status, 18, lim)) ok = false;
    const int rank = (int)cluster_ctarank();
    const int r0 = row_lo(rank), rows = row_lo(rank + 1) - r0;
    const float* red = reinterpret_cast<const float*>(gbase + L::kRing);
    constexpr int chunks = BN / 4;
    // thread t: row t % 64 (at most 64 rows once K is split; consecutive
    // threads take consecutive n, so the fp16 stores coalesce), 4-column
    // chunks t / 64, t / 64 + slots, ...; the S partial loads of a chunk are
    // unrolled (predicated on S) so they are all in flight together
    constexpr int slots = kThreadsW / 64;
    const int lr = threadIdx.x & 63;
    // debug library: the S partial rows this thread reads lie in the receive area
    const bool red_ok = lr >= rows || dcheck(in_area((int64_t)((S - 1) * maxrows + lr) * L::kRedLd * 4, BN * 4,
                                                     L::kRed),
                                             status, 71);
    dispatch_act(p.act, [&](auto gelu) {
      if (lr >= rows || (int)threadIdx.x >= slots * 64 || !red_ok) return;
      for (int ch = threadIdx.x >> 6; ch < chunks; ch += slots) {
        const int c = 4 * ch;
        if constexpr (I8) {
          // int32 partials: exact sums, then the W8A8 epilogue per output
          const int32_t* redi = reinterpret_cast<const int32_t*>(red);
          int4 acc = *reinterpret_cast<const int4*>(redi + lr * L::kRedLd + c);
#pragma unroll
          for (int q = 1; q < 8; ++q) {
            if (q < S) {
              const int4 v = *reinterpret_cast<const int4*>(redi + (q * maxrows + lr) * L::kRedLd + c);
              acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
            }
          }
          const int nn = ta * 128 + r0 + lr;
          if (nn < p.N) {
            const int a4[4] = {acc.x, acc.y, acc.z, acc.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int m = tb * BN + c + j;
              if (m < p.M)
                store_i8_out(p.y_any, p.out_dtype, (int64_t)m * p.ldy + nn, a4[j],
                             p.x_scale ? __ldg(p.x_scale + m) : 0.0f, sWs[lr], sBias[lr]);
            }
          }
          continue;
        }
        float4 acc = *reinterpret_cast<const float4*>(red + lr * L::kRedLd + c);
#pragma unroll
        for (int q = 1; q < 8; ++q) {
          if (q < S) {
            const float4 v = *reinterpret_cast<const float4*>(red + (q * maxrows + lr) * L::kRedLd + c);
            acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
          }
        }
        const int nn = ta * 128 + r0 + lr;
        if (nn < p.N) {
          const float sc = sWs[lr], b = sBias[lr];
          float a4[4] = {fmaf(acc.x, sc, b), fmaf(acc.y, sc, b), fmaf(acc.z, sc, b), fmaf(acc.w, sc, b)};
          apply_act_c<decltype(gelu)::value>(a4);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int m = tb * BN + c + j;
            if (m < p.M) p.y[(int64_t)m * p.ldy + nn] = __float2half_rn(a4[j]);
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
// Host side
// ---------------------------------------------------------------------------
template <int BN, bool W4, int STAGES, int ASTAGES, int MINB, bool SPLITK, bool I8 = false>
static qg_status run_wonly(const CUtensorMap& tmX, const CUtensorMap& tmW, const CUtensorMap& tmS,
                           const CUtensorMap& tmZ, WOnlyParams p, cudaStream_t s) {
  using L = WOnlyLayout<BN, W4, STAGES, ASTAGES, SPLITK, I8>;
  // MINB CTAs must fit one SM: 228 KB of shared memory (1 KB reserved per CTA)
  // and 512 TMEM columns.
  static_assert(MINB * (L::kTotal + 1024) <= 233472, "shared memory does not fit the residency");
  static_assert(MINB * L::kTmemCols <= 512, "tensor memory does not fit the residency");
  static_assert(L::kTotal <= 232448, "above the per-block shared memory limit");
  auto kern = wonly_kernel<BN, W4, STAGES, ASTAGES, MINB, SPLITK, I8>;
  static PerDeviceOnce attr;
  qg_status st = attr.run([&](int) {
    return check_cuda(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kTotal),
                      "cudaFuncSetAttribute(weight-only)");
  });
  if (st != QG_OK) return st;
  if (!SPLITK) p.splits = 1;
  LaunchCfg lc((unsigned)(p.tiles_a * p.tiles_b * p.splits), wonly_threads(BN), L::kTotal, s,
               (unsigned)p.splits);
  return check_cuda(cudaLaunchKernelEx(&lc.cfg, kern, tmX, tmW, tmS, tmZ, p), "weight-only launch");
}

template <bool W4>
static qg_status launch_wonly(const void* x, int64_t ldx, const void* w, int64_t ldw_bytes,
                              const void* scale, const void* zero, const float* ws,
                              const float* bias, void* y, int64_t ldy, int64_t M, int64_t N,
                              int64_t K, cudaStream_t s, int act, bool sym = false, unsigned flags = 0) {
  WOnlyParams p = {};
  p.static_w = (flags & QG_FLAG_STATIC_WEIGHTS) ? 1 : 0;
  p.act = act;
  p.sym = sym ? 1 : 0;
  p.M = (int)M;
  p.N = (int)N;
  p.K = (int)K;
  p.nkb = (int)((K + kKB - 1) / kKB);
  p.w_scale = ws;
  p.bias = bias;
  p.y = static_cast<__half*>(y);
  p.ldy = ldy;
  // Token tile width: 16/32/64 rows for decode batches; above 64 rows the
  // wide-tile kernel (qg_gemm_wonly_wide.cu) dequantizes each weight once per
  // 128 or 256 tokens.  The QG_WONLY_BN switch forces a width (16/32/64 keep
  // these tiles for any M).
  int bn = M <= 16 ? 16 : M <= 32 ? 32 : 64;
  const int bn_env = tuning(kTuneWonlyBn);
  if (bn_env == 16 || bn_env == 32 || bn_env == 64) {
    bn = bn_env;
  } else if (M > 64 || bn_env == 128 || bn_env == 256) {
    return launch_wonly_wide(W4, x, ldx, w, ldw_bytes, scale, zero, ws, bias, y, ldy, M, N, K, s, act, sym, flags,
                             bn_env);
  }
  p.tiles_a = (int)((N + 127) / 128);
  p.tiles_b = (int)((M + bn - 1) / bn);
  // CTAs resident per SM for this tile width (see the dispatch table below);
  // K is split across clusters only while every CTA still gets a slot at once.
  const int minb = bn <= 32 ? 2 : 1;
  const int resident = minb * sm_count();
  const int tiles = p.tiles_a * p.tiles_b;
  int splits = tuning(W4 ? kTuneW4A16Splits : kTuneW8A16Splits);
  if (splits <= 0) {
    splits = 1;
    while (splits < 8 && tiles * (splits + 1) <= resident && splits + 1 <= p.nkb) ++splits;
  }
  if (splits > p.nkb) splits = p.nkb;
  if (splits > 8) splits = 8;
  p.splits = splits;
  p.dbg_wait_us = take_debug_injection(QG_DEBUG_WEIGHT_ONLY);
  p.dbg_withhold = p.dbg_wait_us != 0;

  CUtensorMap tmX, tmW, tmS, tmZ;
  qg_status st;
  if ((st = make_tmap_2d(&tmX, x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, (uint64_t)K, (uint64_t)M,
                         (uint64_t)ldx, 64, (uint32_t)bn, CU_TENSOR_MAP_SWIZZLE_128B)) != QG_OK)
    return st;
  if (W4) {
    if ((st = make_tmap_2d(&tmW, w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)(K / 2), (uint64_t)N,
                           (uint64_t)ldw_bytes, 64, 128, CU_TENSOR_MAP_SWIZZLE_64B)) != QG_OK)
      return st;
    if ((st = make_tmap_2d(&tmS, scale, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, (uint64_t)N,
                           (uint64_t)(K / 64), (uint64_t)N, 128, 2, CU_TENSOR_MAP_SWIZZLE_NONE)) != QG_OK)
      return st;
    if (sym) {
      tmZ = tmS;  // never loaded
    } else if ((st = make_tmap_2d(&tmZ, zero, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, (uint64_t)N,
                                  (uint64_t)(K / 64), (uint64_t)N, 128, 2, CU_TENSOR_MAP_SWIZZLE_NONE)) != QG_OK) {
      return st;
    }
  } else {
    if ((st = make_tmap_2d(&tmW, w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)K, (uint64_t)N,
                           (uint64_t)ldw_bytes, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B)) != QG_OK)
      return st;
    tmS = tmW;
    tmZ = tmW;
  }
  //               BN   W4    STAGES ASTAGES MINB SPLITK
  switch (bn) {
    case 16: return W4 ? run_wonly<16, true, 6, 3, 2, true>(tmX, tmW, tmS, tmZ, p, s)
                       : run_wonly<16, false, 4, 3, 2, true>(tmX, tmW, tmS, tmZ, p, s);
    case 32: return W4 ? run_wonly<32, true, 4, 3, 2, true>(tmX, tmW, tmS, tmZ, p, s)
                       : run_wonly<32, false, 2, 3, 2, true>(tmX, tmW, tmS, tmZ, p, s);
    default: return W4 ? run_wonly<64, true, 6, 3, 1, true>(tmX, tmW, tmS, tmZ, p, s)
                       : run_wonly<64, false, 4, 3, 1, true>(tmX, tmW, tmS, tmZ, p, s);
  }
}

// W4A8 for decode batches (M <= 64) on this pipeline: the int4 codes are
// unpacked to int8 straight into the tensor-memory A operand and multiplied by
// the int8 X codes on the int8 tensor path (tcgen05 kind::i8, A from tensor
// memory), with the W8A8 epilogue.  Same tiles, clusters and split rule as the
// weight-only decode shapes; two CTAs per SM at every tile width.
qg_status launch_w4a8_decode(const int8_t* xq, int64_t ldx, const int32_t* qweight, const float* xs,
                             const float* ws, const float* bias, void* y, int dtype, int64_t ldy, int64_t M,
                             int64_t N, int64_t K, cudaStream_t s) {
  WOnlyParams p = {};
  p.M = (int)M;
  p.N = (int)N;
  p.K = (int)K;
  p.nkb = (int)((K + kKB - 1) / kKB);
  p.w_scale = ws;
  p.bias = bias;
  p.x_scale = xs;
  p.y_any = y;
  p.ldy = ldy;
  p.out_dtype = dtype;
  p.sym = 1;
  const int bn = M <= 16 ? 16 : M <= 32 ? 32 : 64;
  p.tiles_a = (int)((N + 127) / 128);
  p.tiles_b = (int)((M + bn - 1) / bn);
  const int resident = 2 * sm_count();
  const int tiles = p.tiles_a * p.tiles_b;
  int splits = 1;
  while (splits < 8 && tiles * (splits + 1) <= resident && splits + 1 <= p.nkb) ++splits;
  p.splits = splits;
  CUtensorMap tmX, tmW;
  qg_status st;
  // int8 X: one 128-byte swizzle atom per row and K block
  if ((st = make_tmap_2d(&tmX, xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)K, (uint64_t)M, (uint64_t)ldx, kKB,
                         (uint32_t)bn, CU_TENSOR_MAP_SWIZZLE_128B)) != QG_OK)
    return st;
  if ((st = make_tmap_2d(&tmW, qweight, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)(K / 2), (uint64_t)N,
                         (uint64_t)(K / 2), 64, 128, CU_TENSOR_MAP_SWIZZLE_64B)) != QG_OK)
    return st;
  //                               BN   W4    STAGES ASTAGES MINB SPLITK I8
  switch (bn) {
    case 16: return run_wonly<16, true, 8, 3, 2, true, true>(tmX, tmW, tmW, tmW, p, s);
    case 32: return run_wonly<32, true, 6, 3, 2, true, true>(tmX, tmW, tmW, tmW, p, s);
    default: return run_wonly<64, true, 4, 3, 2, true, true>(tmX, tmW, tmW, tmW, p, s);
  }
}

qg_status launch_w8a16(const void* x, int64_t ldx, const int8_t* wq, int64_t ldw, const float* ws,
                       const float* bias, void* y, int64_t ldy, int64_t M, int64_t N, int64_t K,
                       cudaStream_t s, int act, unsigned flags) {
  return launch_wonly<false>(x, ldx, wq, ldw, nullptr, nullptr, ws, bias, y, ldy, M, N, K, s, act, false, flags);
}

qg_status launch_w4a16(const void* x, int64_t ldx, const int32_t* qweight, const void* scale,
                       const void* zero, const float* bias, void* y, int64_t ldy, int64_t M,
                       int64_t N, int64_t K, cudaStream_t s, int act, unsigned flags) {
  return launch_wonly<true>(x, ldx, qweight, K / 2, scale, zero, nullptr, bias, y, ldy, M, N, K, s, act, false,
                            flags);
}

qg_status launch_w4a16_sym(const void* x, int64_t ldx, const int32_t* qweight, const void* scale,
                           const float* bias, void* y, int64_t ldy, int64_t M, int64_t N, int64_t K,
                           cudaStream_t s, int act) {
  return launch_wonly<true>(x, ldx, qweight, K / 2, scale, nullptr, nullptr, bias, y, ldy, M, N, K, s, act,
                            true);
}

}  // namespace qg

// qg_gemm_decode.cu -- stream-K decode GEMMs (M <= 64) on the sm_100a tensor
// cores, for all three forms of the hot path:
//
//   I8 (W8A8):  Y = float(sum Xq*Wq) * x_scale[m] * w_scale[n] + bias[n]
//   W8 (W8A16): Y = w_scale[n] * sum X*Wq + bias[n]
//   W4 (W4A16): Y = sum X*(q - z)*s + bias[n]
//
// Pages: "量化算法的本质" (W8A8, W8A16/W4A16), "量化与多精度算子" §四 (int32 /
// fp32 accumulation, dequant at the end or on chip), "INT4/FP16混合精度GEMM"
// §3.2 §4.2 (unpack, (q - zp) * scale, fp16 matmul with fp32 accumulation).
//
// Decode GEMMs stream the weight matrix once through the tensor cores; the
// time is the weight bytes over HBM bandwidth plus fill and drain.  This
// kernel runs one CTA per SM and gives every CTA the same number of
// (tile, K block) iterations -- tile = 128 weight rows (the TMEM lanes), K
// block = 128 elements -- taken in order, so each CTA streams one contiguous
// range that may start and end inside a tile ("stream-K").  A tile finished
// by one CTA goes straight to the epilogue; a tile shared by several CTAs has
// each contributor write its partial accumulator to the caller's workspace,
// and the last contributor (per 32-row quadrant, found with an atomic ticket)
// adds the partials in contributor order and writes Y.  Every SM does the same
// work, with no cluster barrier waiting for the slowest member.
//
// Warps: 0 TMA producer; 1..NI MMA issuers (the per-instruction issue cost of
// a narrow MMA is per issuing thread, so decode tiles use several, each into
// its own TMEM accumulator); NI+1..NI+4 epilogue (one per TMEM lane quadrant,
// double-buffered accumulator); then, for W8/W4, 16 converter warps that
// dequantize into a TMEM A-operand ring (four per lane quadrant, one per
// 32-element quarter of a K block).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "qg_dequant.cuh"
#include "qg_device.cuh"
#include "qg_internal.h"

namespace qg {

static __device__ unsigned long long g_status_decode;

unsigned long long read_clear_status_decode(cudaStream_t s) {
  unsigned long long v = 0, z = 0;
  cudaMemcpyFromSymbolAsync(&v, g_status_decode, sizeof(v), 0, cudaMemcpyDeviceToHost, s);
  cudaMemcpyToSymbolAsync(g_status_decode, &z, sizeof(z), 0, cudaMemcpyHostToDevice, s);
  cudaStreamSynchronize(s);
  return v;
}

enum DecKind { kDecI8 = 0, kDecW8 = 1, kDecW4 = 2 };
constexpr int kDKB = 128;  // K elements per block (bytes for int8 operands)

struct DecodeParams {
  int M, N, K;
  int tiles, nkb, iters;  // tiles of 128 weight rows, K blocks, tiles * nkb
  const float* x_scale;   // I8
  const float* w_scale;   // I8, W8
  const float* bias;
  void* y;
  int64_t ldy;
  int out_dtype;          // I8: any qg_dtype; W8/W4: QG_F16
  uint32_t* partial;      // [grid][2][128][BN] 32-bit partial accumulators
  uint32_t* ticket;       // [kMaxDecGrid][4] arrival counters (zero between launches)
  // Fault injection for tests (qg_debug_inject_timeout), zero in every other
  // launch: withhold (1) the copy of CTA 0's first K block, and bound every
  // wait by dbg_wait_us microseconds instead of kWaitLimitNs (0).
  int dbg_withhold;
  uint32_t dbg_wait_us;
};

// Workspace layout, independent of the problem so that one zero-filled buffer
// serves every shape: kMaxDecGrid x 4 tickets at offset 0, then the partials.
// A tile shared by several CTAs is the last segment of its first contributor,
// so its tickets are indexed by that CTA (and the quadrant).
constexpr int kMaxDecGrid = 1024;
constexpr size_t kTicketBytes = (size_t)kMaxDecGrid * 4 * 4;

__host__ __device__ constexpr int dec_issuers(int bn) { return bn <= 16 ? 4 : (bn <= 32 ? 2 : 1); }
__host__ __device__ constexpr int dec_conv_warps(int kind) { return kind == kDecI8 ? 0 : 16; }
__host__ __device__ constexpr int dec_threads(int kind, int bn) {
  return 32 * (1 + dec_issuers(bn) + 4 + dec_conv_warps(kind));
}

template <int KIND, int BN, int STAGES, int ASTAGES>
struct DecLayout {
  static constexpr bool kConv = KIND != kDecI8;
  static constexpr int kX = KIND == kDecI8 ? BN * 128 : BN * 256;  // B operand (X) bytes per stage
  static constexpr int kW = KIND == kDecW4 ? 128 * 64 : 128 * 128;  // weight tile bytes
  static constexpr int kSZ = KIND == kDecW4 ? 2 * 128 * 2 : 0;      // fp16 scale (and zero) tile
  static constexpr int kStage = kX + kW + 2 * kSZ;
  static constexpr int kRing = STAGES * kStage;
  static constexpr int kBars = (2 * STAGES + 2 * ASTAGES + 5) * 8 + 16;
  static constexpr int kTotal = 1024 + kRing + kBars;
  static constexpr int kNI = dec_issuers(BN);
  static constexpr int kAccCols = kNI * BN;                          // one accumulator per issuer
  static constexpr int kDCols = 2 * (kAccCols < 64 ? 64 : kAccCols);  // two accumulator buffers
  static constexpr int kNeed = kDCols + (kConv ? 64 * ASTAGES : 0);
  static constexpr int kTmemCols = kNeed <= 32 ? 32 : kNeed <= 64 ? 64 : kNeed <= 128 ? 128 : kNeed <= 256 ? 256 : 512;
  static_assert(kStage % 1024 == 0, "stage must keep 1024-byte alignment");
  static_assert(kNeed <= 512, "tensor memory overflow");
  static_assert(!kConv || (STAGES % 4 == 0 && ASTAGES % 4 == 0),
                "ring lengths must be multiples of the four converter groups");
  static_assert(kTotal <= 232448, "shared memory overflow");
};

// ---- the stream-K partition -------------------------------------------------
// CTA c owns iterations [first_iter(c), first_iter(c+1)) of tiles*nkb, in
// tile-major order.
__device__ __forceinline__ int first_iter(int c, int iters, int grid) {
  return (int)(((unsigned)c * (unsigned)iters) / (unsigned)grid);  // iters * grid < 2^31 (host check)
}

// The CTA that owns iteration i.
__device__ __forceinline__ int owner_cta(int i, int iters, int grid) {
  int c = (int)(((unsigned)i * (unsigned)grid) / (unsigned)iters);
  while (c + 1 < grid && first_iter(c + 1, iters, grid) <= i) ++c;
  while (c > 0 && first_iter(c, iters, grid) > i) --c;
  return c;
}

template <int KIND>
__device__ __forceinline__ void dec_store(void* y, int dtype, int64_t idx, float v, int32_t raw) {
  if (KIND != kDecI8) {
    static_cast<__half*>(y)[idx] = __float2half_rn(v);
  } else {
    switch (dtype) {
      case QG_F32: static_cast<float*>(y)[idx] = v; break;
      case QG_F16: static_cast<__half*>(y)[idx] = __float2half_rn(v); break;
      case QG_BF16: static_cast<__nv_bfloat16*>(y)[idx] = __float2bfloat16_rn(v); break;
      default: static_cast<int32_t*>(y)[idx] = raw; break;
    }
  }
}

template <int KIND, int BN, int STAGES, int ASTAGES>
__global__ void __launch_bounds__(dec_threads(KIND, BN), 1)
    decode_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                  const __grid_constant__ CUtensorMap tmS, const __grid_constant__ CUtensorMap tmZ,
                  const DecodeParams p) {
  using L = DecLayout<KIND, BN, STAGES, ASTAGES>;
  constexpr int NI = L::kNI;
  constexpr int kConvW = dec_conv_warps(KIND);
  constexpr int kEpi0 = 1 + NI;     // first epilogue warp
  constexpr int kConv0 = kEpi0 + 4;  // first converter warp
  constexpr uint32_t kIdesc = KIND == kDecI8 ? idesc_i8_s32(128, BN) : idesc_f16_f32(128, BN);
  constexpr int kStepsPerBlock = KIND == kDecI8 ? kDKB / 32 : kDKB / 16;  // MMAs per K block
  constexpr int kBufCols = L::kDCols / 2;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_base = smem_u32(smem_raw);
  const uint32_t base = (raw_base + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw_base);
  const uint32_t bars = base + L::kRing;
  auto raw_full = [&](int s) { return bars + 8u * s; };
  auto raw_empty = [&](int s) { return bars + 8u * (STAGES + s); };
  auto a_full = [&](int a) { return bars + 8u * (2 * STAGES + a); };
  auto a_empty = [&](int a) { return bars + 8u * (2 * STAGES + ASTAGES + a); };
  auto d_full = [&](int b) { return bars + 8u * (2 * STAGES + 2 * ASTAGES + b); };
  auto d_empty = [&](int b) { return bars + 8u * (2 * STAGES + 2 * ASTAGES + 2 + b); };
  const uint32_t done_bar = bars + 8u * (2 * STAGES + 2 * ASTAGES + 4);  // every warp finished
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + L::kRing + (2 * STAGES + 2 * ASTAGES + 5) * 8);
  auto stage_x = [&](int s) { return base + (uint32_t)(s * L::kStage); };
  auto stage_w = [&](int s) { return base + (uint32_t)(s * L::kStage + L::kX); };
  auto stage_sc = [&](int s) { return base + (uint32_t)(s * L::kStage + L::kX + L::kW); };
  auto stage_ze = [&](int s) { return base + (uint32_t)(s * L::kStage + L::kX + L::kW + L::kSZ); };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  unsigned long long* status = &g_status_decode;
  const uint64_t lim = p.dbg_wait_us ? (uint64_t)p.dbg_wait_us * 1000ull : kWaitLimitNs;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(raw_full(s), 1);
      mbar_init(raw_empty(s), (L::kConv ? 4 : 0) + NI);  // one converter group (weights) + issuer commits (X)
    }
    for (int a = 0; a < ASTAGES; ++a) {
      mbar_init(a_full(a), 4);
      mbar_init(a_empty(a), NI);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(d_full(b), NI);
      mbar_init(d_empty(b), 4);  // one arrive per epilogue warp
    }
    mbar_init(done_bar, dec_threads(KIND, BN) / 32);
    fence_mbar_init();
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmW);
    if (KIND == kDecW4) {
      tma_prefetch_desc(&tmS);
      tma_prefetch_desc(&tmZ);
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
  pdl_trigger();
  pdl_wait();  // inputs of the preceding kernel are visible from here on

  const int G = gridDim.x;
  const int it0 = first_iter(blockIdx.x, p.iters, G);
  const int it1 = first_iter(blockIdx.x + 1, p.iters, G);
  const int t_first = it0 / p.nkb;
  bool ok = true;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_x = policy_evict_last();
      int it = 0;
      for (int t = t_first; t * p.nkb < it1 && ok; ++t) {
        const int kb0 = max(it0 - t * p.nkb, 0), kb1 = min(it1 - t * p.nkb, p.nkb);
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if (!mbar_wait(raw_empty(s), ph ^ 1u, status, 21, lim)) { ok = false; break; }
          if (p.dbg_withhold && blockIdx.x == 0 && it == 0) continue;  // test-only: this stage never lands
          mbar_arrive_expect_tx(raw_full(s), (uint32_t)L::kStage);
          if (KIND == kDecI8) {
            if (tma_ok(stage_x(s), kb * kDKB, (KIND == kDecI8 ? 1 : 2), status, 60))
              tma_load_2d_hint(stage_x(s), &tmX, raw_full(s), kb * kDKB, 0, pol_x);
          } else {
            if (tma_ok(stage_x(s), kb * kDKB, (KIND == kDecI8 ? 1 : 2), status, 61))
              tma_load_2d_hint(stage_x(s), &tmX, raw_full(s), kb * kDKB, 0, pol_x);
            if (tma_ok(stage_x(s) + BN * 128, kb * kDKB + 64, (KIND == kDecI8 ? 1 : 2), status, 62))
              tma_load_2d_hint(stage_x(s) + BN * 128, &tmX, raw_full(s), kb * kDKB + 64, 0, pol_x);
          }
          if (KIND == kDecW4) {
            if (tma_ok(stage_w(s), kb * (kDKB / 2), 1, status, 63))
              tma_load_2d_hint(stage_w(s), &tmW, raw_full(s), kb * (kDKB / 2), t * 128, pol_w);
            if (tma_ok(stage_sc(s), t * 128, 2, status, 64))
              tma_load_2d_hint(stage_sc(s), &tmS, raw_full(s), t * 128, kb * 2, pol_w);
            if (tma_ok(stage_ze(s), t * 128, 2, status, 65))
              tma_load_2d_hint(stage_ze(s), &tmZ, raw_full(s), t * 128, kb * 2, pol_w);
          } else {
            if (tma_ok(stage_w(s), kb * kDKB, 1, status, 66))
              tma_load_2d_hint(stage_w(s), &tmW, raw_full(s), kb * kDKB, t * 128, pol_w);
          }
        }
      }
      // Wait (bounded) until every load this thread issued has landed, so that
      // no copy into this CTA's shared memory outlives it, whether or not the
      // consumers got to them (they may have given up).  After a normal run
      // these phases are complete and each wait is one poll.
      for (int i = it - 1; i >= 0 && i >= it - STAGES; --i) {
        if (p.dbg_withhold && blockIdx.x == 0 && i == 0) continue;  // never issued
        mbar_wait(raw_full(i % STAGES), (uint32_t)(i / STAGES) & 1u, status, 29, lim);
      }
    }
  } else if (warp < kEpi0) {
    // ---------------- MMA issuers ----------------
    const int iss = warp - 1;
    if (lane == 0) {
      int it = 0, seg = 0;
      for (int t = t_first; t * p.nkb < it1 && ok; ++t, ++seg) {
        const int kb0 = max(it0 - t * p.nkb, 0), kb1 = min(it1 - t * p.nkb, p.nkb);
        const int buf = seg & 1;
        if (!mbar_wait(d_empty(buf), (uint32_t)((seg >> 1) & 1) ^ 1u, status, 22, lim)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(buf * kBufCols + iss * BN);
        bool first = true;
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if (!mbar_wait(raw_full(s), ph, status, 23, lim)) { ok = false; break; }
          if (KIND != kDecI8) {
            const int a = it % ASTAGES;
            if (!mbar_wait(a_full(a), (uint32_t)(it / ASTAGES) & 1u, status, 24, lim)) { ok = false; break; }
          }
          tc_fence_after();
          if (KIND == kDecI8) {
            const uint64_t da = sdesc_sw128(stage_w(s));
            const uint64_t db = sdesc_sw128(stage_x(s));
#pragma unroll
            for (int k = iss; k < kStepsPerBlock; k += NI) {
              mma_i8(d, da + 2u * k, db + 2u * k, kIdesc, first ? 0u : 1u);
              first = false;
            }
          } else {
            const int a = it % ASTAGES;
            const uint32_t a_col = tmem + (uint32_t)(L::kDCols + 64 * a);
#pragma unroll
            for (int j = iss; j < kStepsPerBlock; j += NI) {
              const uint64_t db = sdesc_sw128(stage_x(s) + (uint32_t)((j >> 2) * BN * 128 + (j & 3) * 32));
              mma_f16_ts(d, a_col + 8u * j, db, kIdesc, first ? 0u : 1u);
              first = false;
            }
            mma_commit(a_empty(a));
          }
          mma_commit(raw_empty(s));
        }
        if (!ok) break;
        mma_commit(d_full(buf));
      }
    }
  } else if (warp < kConv0) {
    // ---------------- epilogue (one warp per TMEM lane quadrant) ----------------
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    const bool scaled = KIND != kDecI8 || p.out_dtype != QG_I32;
    float xs[BN];
    if (KIND == kDecI8) {
#pragma unroll
      for (int j = 0; j < BN; ++j) xs[j] = (scaled && j < p.M) ? __ldg(p.x_scale + j) : 0.0f;
    }
    int seg = 0;
    for (int t = t_first; t * p.nkb < it1 && ok; ++t, ++seg) {
      const int kb0 = max(it0 - t * p.nkb, 0), kb1 = min(it1 - t * p.nkb, p.nkb);
      const int buf = seg & 1;
      const int n = t * 128 + row;
      const bool nvalid = n < p.N;
      const float ws = (KIND != kDecW4 && scaled && nvalid) ? __ldg(p.w_scale + n) : 1.0f;
      const float bias = (p.bias && nvalid) ? __ldg(p.bias + n) : 0.0f;
      // contributors of this tile (computed while the mainloop runs)
      const int c_first = owner_cta(t * p.nkb, p.iters, G);
      const int c_last = owner_cta(t * p.nkb + p.nkb - 1, p.iters, G);
      if (!mbar_wait(d_full(buf), (uint32_t)((seg >> 1) & 1), status, 25, lim)) { ok = false; break; }
      tc_fence_after();
      // sum the issuers' accumulators (int32 exactly, fp32 in issuer order)
      uint32_t acc[BN];
#pragma unroll
      for (int c0 = 0; c0 < BN; c0 += 16) {
        uint32_t r[16];
        tmem_ld16(tmem + lane_addr + (uint32_t)(buf * kBufCols + c0), r);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j) acc[c0 + j] = r[j];
#pragma unroll
        for (int a = 1; a < NI; ++a) {
          tmem_ld16(tmem + lane_addr + (uint32_t)(buf * kBufCols + a * BN + c0), r);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            if (KIND == kDecI8) acc[c0 + j] = (uint32_t)((int32_t)acc[c0 + j] + (int32_t)r[j]);
            else acc[c0 + j] = __float_as_uint(__uint_as_float(acc[c0 + j]) + __uint_as_float(r[j]));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(d_empty(buf));  // the accumulator buffer may be reused

      bool finish = true;
      if (c_first != c_last) {
        // Partial tile.  If every other contributor has already published
        // (ticket == n - 1, read with acquire), this CTA is last: it adds the
        // others' rows to its own accumulator directly.  Otherwise it
        // publishes its rows and takes a ticket; the ticket holder that brings
        // the count to n - 1... n is last and does the sum.
        const uint32_t need = (uint32_t)(c_last - c_first);
        uint32_t* tk = p.ticket + c_first * 4 + quad;
        uint32_t seen = 0;
        if (lane == 0) seen = ld_acquire_gpu(tk);
        seen = __shfl_sync(0xffffffffu, seen, 0);
        __syncwarp();
        finish = seen == need;
        bool own_published = false;
        if (!finish) {
          const int slot = (t == t_first) ? 0 : 1;
          uint32_t* mine = p.partial + (((size_t)blockIdx.x * 2 + slot) * 128 + row) * BN;
#pragma unroll
          for (int j = 0; j < BN; j += 4)
            __stcg(reinterpret_cast<uint4*>(mine + j), make_uint4(acc[j], acc[j + 1], acc[j + 2], acc[j + 3]));
          fence_acq_rel_gpu();  // this lane's rows before the ticket
          __syncwarp();
          uint32_t ticket = 0;
          if (lane == 0) ticket = atom_add_acq_rel_gpu(tk, 1u);
          ticket = __shfl_sync(0xffffffffu, ticket, 0);
          __syncwarp();
          finish = ticket == need;
          own_published = true;
        }
        if (finish) {
          // last arrival: every contributor's rows are visible; add them in
          // contributor order (deterministic), then reset the ticket
          // Loads of up to kBatch contributors are issued together (their L2
          // latencies overlap), then added in contributor order; this CTA's own
          // rows come from its registers when it did not publish them.
          uint32_t mine_acc[BN];
#pragma unroll
          for (int j = 0; j < BN; ++j) mine_acc[j] = acc[j];
          (void)own_published;
          // (W8/W4 CTAs run 22-25 warps, so fewer registers per thread: smaller batches)
          constexpr int kBatch = KIND == kDecI8 ? (BN <= 16 ? 8 : (BN <= 32 ? 4 : 2)) : (BN <= 16 ? 2 : 1);
          for (int c0 = c_first; c0 <= c_last; c0 += kBatch) {
            uint4 v[kBatch][BN / 4];
#pragma unroll
            for (int b = 0; b < kBatch; ++b) {
              const int cc = c0 + b;
              if (cc <= c_last && cc != (int)blockIdx.x) {
                const int sl = (t == first_iter(cc, p.iters, G) / p.nkb) ? 0 : 1;
                const uint4* src = reinterpret_cast<const uint4*>(p.partial + (((size_t)cc * 2 + sl) * 128 + row) * BN);
#pragma unroll
                for (int j = 0; j < BN / 4; ++j) v[b][j] = __ldcg(src + j);
              }
            }
#pragma unroll
            for (int b = 0; b < kBatch; ++b) {
              const int cc = c0 + b;
              if (cc <= c_last) {
#pragma unroll
                for (int j = 0; j < BN / 4; ++j) {
                  uint32_t vv[4] = {v[b][j].x, v[b][j].y, v[b][j].z, v[b][j].w};
                  if (cc == (int)blockIdx.x) {
                    vv[0] = mine_acc[4 * j]; vv[1] = mine_acc[4 * j + 1];
                    vv[2] = mine_acc[4 * j + 2]; vv[3] = mine_acc[4 * j + 3];
                  }
#pragma unroll
                  for (int e = 0; e < 4; ++e) {
                    uint32_t& a = acc[4 * j + e];
                    if (cc == c_first) a = vv[e];
                    else if (KIND == kDecI8) a = (uint32_t)((int32_t)a + (int32_t)vv[e]);
                    else a = __float_as_uint(__uint_as_float(a) + __uint_as_float(vv[e]));
                  }
                }
              }
            }
          }
          if (lane == 0) atomicExch(p.ticket + c_first * 4 + quad, 0u);
        }
      }
      if (finish && nvalid) {
#pragma unroll
        for (int j = 0; j < BN; ++j) {
          if (j < p.M) {
            const float v = KIND == kDecI8 ? fmaf((float)(int32_t)acc[j], xs[j] * ws, bias)
                                           : fmaf(__uint_as_float(acc[j]), ws, bias);
            dec_store<KIND>(p.y, p.out_dtype, (int64_t)j * p.ldy + n, v, (int32_t)acc[j]);
          }
        }
      }
      (void)kb0;
      (void)kb1;
    }
  } else if (L::kConv) {
    // ---------------- converters (W8 / W4) ----------------
    // Four groups of four warps (one warp per TMEM lane quadrant) take turns
    // over this CTA's K blocks; each warp converts a whole 128-wide block of its
    // 32 rows.  Ring lengths are multiples of four, so every shared-memory and
    // tensor-memory stage belongs to one group.
    const int cw = warp - kConv0;      // 0..15
    const int quad = warp & 3;         // TMEM lane quadrant this warp may access
    const int grp = cw >> 2;           // converter group
    const int row = quad * 32 + lane;  // TMEM lane = weight row within the tile
    const int gt = (cw & 3) * 32 + lane;  // thread within the group
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    int it = 0;
    int s = grp, a = grp;
    uint32_t ph = 0, aph = 0;
    for (int t = t_first; t * p.nkb < it1 && ok; ++t) {
      const int kb0 = max(it0 - t * p.nkb, 0), kb1 = min(it1 - t * p.nkb, p.nkb);
      for (int kb = kb0; kb < kb1; ++kb, ++it) {
        if ((it & 3) != grp) continue;
        if (!mbar_wait(raw_full(s), ph, status, 26, lim)) { ok = false; break; }
        if (!mbar_wait(a_empty(a), aph ^ 1u, status, 27, lim)) { ok = false; break; }
        tc_fence_after();
        const uint32_t dst = tmem + lane_addr + (uint32_t)(L::kDCols + 64 * a);
        if (KIND == kDecW4) {
          uint8_t* xst = gbase + (stage_x(s) - base);
          for (int c = gt; c < BN * 16; c += 128) permute_x_chunk(xst + 16 * c);
          fence_proxy_async_smem();
          const uint8_t* wrow = gbase + (stage_w(s) - base) + row * 64;
          const __half* sc = reinterpret_cast<const __half*>(gbase + (stage_sc(s) - base));
          const __half* ze = reinterpret_cast<const __half*>(gbase + (stage_ze(s) - base));
#pragma unroll
          for (int g = 0; g < 2; ++g) {
            uint32_t s2, c_lo, c_hi;
            u4_group_consts(__half_as_ushort(sc[g * 128 + row]), __half_as_ushort(ze[g * 128 + row]), s2, c_lo,
                            c_hi);
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
              const int chunk = 2 * g + cc;
              const uint4 v = *reinterpret_cast<const uint4*>(wrow + ((chunk ^ ((row >> 1) & 3)) << 4));
              const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
              uint32_t r[16];
#pragma unroll
              for (int i = 0; i < 4; ++i) u4x8_to_h2x4(wv[i], s2, c_lo, c_hi, 0x64006400u, 0x64006400u, r + 4 * i);
              tmem_st16(dst + 16 * chunk, r);
            }
          }
        } else {
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
        if ((s += 4) >= STAGES) { s -= STAGES; ph ^= 1u; }
        if ((a += 4) >= ASTAGES) { a -= ASTAGES; aph ^= 1u; }
      }
    }
  }

  // Teardown: each warp reports that it is done with tensor memory; the
  // allocating warp frees it once all have (bounded wait).  Shared memory
  // lives until the last thread of the CTA exits.
  __syncwarp();
  tc_fence_before();
  if (lane == 0) mbar_arrive(done_bar);
  if (warp == 1) {
    if (lane == 0) mbar_wait(done_bar, 0, status, 30, lim);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
static int dec_bn(int64_t M) { return M <= 16 ? 16 : (M <= 32 ? 32 : 64); }

static int dec_grid_cap() { return sm_count() < kMaxDecGrid ? sm_count() : kMaxDecGrid; }

size_t decode_ticket_bytes() { return kTicketBytes; }

size_t decode_workspace_bytes(int64_t M, int64_t N) {
  (void)N;
  return kTicketBytes + (size_t)dec_grid_cap() * 2 * 128 * dec_bn(M) * 4;
}

template <int KIND, int BN, int STAGES, int ASTAGES>
static qg_status run_decode(const CUtensorMap& tmX, const CUtensorMap& tmW, const CUtensorMap& tmS,
                            const CUtensorMap& tmZ, DecodeParams p, int grid, cudaStream_t s) {
  using L = DecLayout<KIND, BN, STAGES, ASTAGES>;
  auto kern = decode_kernel<KIND, BN, STAGES, ASTAGES>;
  static PerDeviceOnce attr;
  qg_status st = attr.run([&](int) {
    return check_cuda(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kTotal),
                      "cudaFuncSetAttribute(decode)");
  });
  if (st != QG_OK) return st;
  LaunchCfg lc((unsigned)grid, dec_threads(KIND, BN), L::kTotal, s);
  return check_cuda(cudaLaunchKernelEx(&lc.cfg, kern, tmX, tmW, tmS, tmZ, p), "decode launch");
}

static qg_status decode_common(int kind, const void* x, int64_t ldx, const void* w, int64_t ldw_bytes,
                               const void* scale, const void* zero, const float* xs,
                               const float* ws, const float* bias, void* y, int dtype, int64_t ldy,
                               int64_t M, int64_t N, int64_t K, void* workspace, cudaStream_t s) {
  const int bn = dec_bn(M);
  DecodeParams p = {};
  p.M = (int)M;
  p.N = (int)N;
  p.K = (int)K;
  p.tiles = (int)((N + 127) / 128);
  p.nkb = (int)((K + kDKB - 1) / kDKB);
  p.iters = p.tiles * p.nkb;
  p.x_scale = xs;
  p.w_scale = ws;
  p.bias = bias;
  p.y = y;
  p.ldy = ldy;
  p.out_dtype = dtype;
  const int grid = dec_grid_cap() < p.iters ? dec_grid_cap() : p.iters;
  if ((int64_t)p.iters * grid >= ((int64_t)1 << 31))
    return fail(QG_ERR_UNSUPPORTED, "decode problem too large for the stream-K partition (%d iterations)", p.iters);
  uint8_t* wsb = static_cast<uint8_t*>(workspace);
  p.ticket = reinterpret_cast<uint32_t*>(wsb);
  p.partial = reinterpret_cast<uint32_t*>(wsb + kTicketBytes);

  CUtensorMap tmX, tmW, tmS, tmZ;
  qg_status st;
  if (kind == kDecI8) {
    if ((st = make_tmap_2d(&tmX, x, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)K, (uint64_t)M,
                           (uint64_t)ldx, kDKB, (uint32_t)bn, CU_TENSOR_MAP_SWIZZLE_128B)) != QG_OK)
      return st;
  } else {
    if ((st = make_tmap_2d(&tmX, x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, (uint64_t)K, (uint64_t)M,
                           (uint64_t)ldx, 64, (uint32_t)bn, CU_TENSOR_MAP_SWIZZLE_128B)) != QG_OK)
      return st;
  }
  if (kind == kDecW4) {
    if ((st = make_tmap_2d(&tmW, w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)(K / 2), (uint64_t)N,
                           (uint64_t)ldw_bytes, 64, 128, CU_TENSOR_MAP_SWIZZLE_64B)) != QG_OK)
      return st;
    if ((st = make_tmap_2d(&tmS, scale, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, (uint64_t)N,
                           (uint64_t)(K / 64), (uint64_t)N, 128, 2, CU_TENSOR_MAP_SWIZZLE_NONE)) != QG_OK)
      return st;
    if ((st = make_tmap_2d(&tmZ, zero, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, (uint64_t)N,
                           (uint64_t)(K / 64), (uint64_t)N, 128, 2, CU_TENSOR_MAP_SWIZZLE_NONE)) != QG_OK)
      return st;
  } else {
    if ((st = make_tmap_2d(&tmW, w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)K, (uint64_t)N,
                           (uint64_t)ldw_bytes, kDKB, 128, CU_TENSOR_MAP_SWIZZLE_128B)) != QG_OK)
      return st;
    tmS = tmW;
    tmZ = tmW;
  }
  p.dbg_wait_us = take_debug_injection(QG_DEBUG_STREAM_K);
  p.dbg_withhold = p.dbg_wait_us != 0;
  //                                      KIND    BN STAGES ASTAGES
  if (kind == kDecI8) {
    if (bn == 16) return run_decode<kDecI8, 16, 10, 1>(tmX, tmW, tmS, tmZ, p, grid, s);
    if (bn == 32) return run_decode<kDecI8, 32, 9, 1>(tmX, tmW, tmS, tmZ, p, grid, s);
    return run_decode<kDecI8, 64, 8, 1>(tmX, tmW, tmS, tmZ, p, grid, s);
  }
  if (kind == kDecW8) {
    if (bn == 16) return run_decode<kDecW8, 16, 8, 4>(tmX, tmW, tmS, tmZ, p, grid, s);
    if (bn == 32) return run_decode<kDecW8, 32, 8, 4>(tmX, tmW, tmS, tmZ, p, grid, s);
    return run_decode<kDecW8, 64, 4, 4>(tmX, tmW, tmS, tmZ, p, grid, s);
  }
  if (bn == 16) return run_decode<kDecW4, 16, 12, 4>(tmX, tmW, tmS, tmZ, p, grid, s);
  if (bn == 32) return run_decode<kDecW4, 32, 8, 4>(tmX, tmW, tmS, tmZ, p, grid, s);
  return run_decode<kDecW4, 64, 8, 4>(tmX, tmW, tmS, tmZ, p, grid, s);
}

qg_status launch_decode_w8a8(const int8_t* xq, int64_t ldx, const int8_t* wq, int64_t ldw,
                             const float* xs, const float* ws, const float* bias, void* y, int dtype,
                             int64_t ldy, int64_t M, int64_t N, int64_t K, void* workspace,
                             cudaStream_t s) {
  return decode_common(kDecI8, xq, ldx, wq, ldw, nullptr, nullptr, xs, ws, bias, y, dtype, ldy, M, N,
                       K, workspace, s);
}

qg_status launch_decode_w8a16(const void* x, int64_t ldx, const int8_t* wq, int64_t ldw,
                              const float* ws, const float* bias, void* y, int64_t ldy, int64_t M,
                              int64_t N, int64_t K, void* workspace, cudaStream_t s) {
  return decode_common(kDecW8, x, ldx, wq, ldw, nullptr, nullptr, nullptr, ws, bias, y, QG_F16, ldy, M,
                       N, K, workspace, s);
}

qg_status launch_decode_w4a16(const void* x, int64_t ldx, const int32_t* qweight, const void* scale,
                              const void* zero, const float* bias, void* y, int64_t ldy, int64_t M,
                              int64_t N, int64_t K, void* workspace, cudaStream_t s) {
  return decode_common(kDecW4, x, ldx, qweight, K / 2, scale, zero, nullptr, nullptr, bias, y, QG_F16,
                       ldy, M, N, K, workspace, s);
}

}  // namespace qg

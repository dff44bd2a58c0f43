// bf16 GEMM C = A W^T on the 5th-generation tensor cores (tcgen05), with the
// block's memory-bound tail fused into the epilogue: bias, GELU-tanh on a
// column range, and the gated residual x + gate * y.
//
// Page: "compile_graph" (chenyy20.com), §1.1 and §2 — the block's linears are
// the large kernels, and the elementwise tail around them is a separate HBM
// round trip unless fused into the producing kernel.
//
// Design (sm_100a):
//   - persistent CTAs, one per SM, tiles of 128 x 256 taken in M-fastest order
//     so the CTAs running together share B tiles in L2 (the SM-pair kernel
//     below picks M- or N-fastest per shape);
//   - warp 0: TMA producer (4-stage ring of 128x64 A and 256x64 B tiles,
//     128-byte swizzle); warp 1: TMEM allocator + single-thread MMA issuer
//     (tcgen05.mma 128x256x16, fp32 accumulators in TMEM); warps 2-5: epilogue
//     (tcgen05.ld -> registers -> fused math -> bf16 stores);
//   - two TMEM accumulators (2 x 256 columns) so the epilogue of tile i
//     overlaps the main loop of tile i+1.
#pragma once

#include "common.cuh"

namespace dit {
namespace gemm {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;  // 64 bf16 = 128 bytes = one swizzle row
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int NUM_THREADS = 192;
constexpr uint32_t TMEM_COLS = 512;
constexpr int BAR_BYTES = 256;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + BAR_BYTES + 1024;  // + alignment slack
constexpr uint32_t IDESC = idesc_bf16(BM, BN, 0, 0);

struct Epi {
  bf16* C;
  int64_t ldc;
  bf16* C2;
  int64_t ldc2;
  int split_col;
  const bf16* bias;
  int gelu_col_begin;
  const float* gate;
  int64_t gate_stride;
  const bf16* resid;
  int64_t ldr;
  int rows_per_batch;
  // fused QK RMSNorm + RoPE on output columns [0, qk_cols) (0 = off):
  // [0, qk_cols/2) are q heads, [qk_cols/2, qk_cols) k heads, 128 columns each
  int qk_cols;
  int qk_norm;
  float qk_eps;
  const bf16* q_scale;
  const bf16* k_scale;
  const float2* rope;  // [rope_rows][64] (cos, sin); row of output row m = m % rope_rows
  int rope_rows;
  // Weight kept in L2 (pair kernel, N-fastest raster, with a persisting L2
  // set-aside): the weight's loads take the evict-last policy, and when a CTA
  // is done it returns its share of [w_keep, w_keep + w_keep_bytes) to normal
  // priority, so the next kernels get the whole L2 back.  nullptr: off.
  const uint8_t* w_keep;
  int64_t w_keep_bytes;
};

// One 128-column head of q or k for output row m: bias, optional RMSNorm with
// its per-dimension scale, rotation of each pair (2p, 2p+1) by the RoPE table,
// bf16 store.  Two passes over TMEM (sum of squares, then transform) keep the
// register footprint at one 32-column chunk.
__device__ __forceinline__ void epilogue_qk_head(uint32_t t_head, int m, int n_head, const Epi& ep, bool row_ok) {
  float ss = 0.0f;
  if (ep.qk_norm) {
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      uint32_t r[32];
      tmem_ld32(t_head + (uint32_t)(c * 32), r);
      const uint4* bp = reinterpret_cast<const uint4*>(ep.bias + n_head + c * 32);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint4 u = ep.bias ? __ldg(bp + q) : make_uint4(0, 0, 0, 0);
        const float b8[8] = {bf16_lo(u.x), bf16_hi(u.x), bf16_lo(u.y), bf16_hi(u.y),
                             bf16_lo(u.z), bf16_hi(u.z), bf16_lo(u.w), bf16_hi(u.w)};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float v = __uint_as_float(r[8 * q + j]) + b8[j];
          ss = fmaf(v, v, ss);
        }
      }
    }
  }
  const float rs = ep.qk_norm ? rsqrtf(ss * (1.0f / 128.0f) + ep.qk_eps) : 1.0f;
  const bool is_k = n_head >= (ep.qk_cols >> 1);
  const bf16* sc = is_k ? ep.k_scale : ep.q_scale;
  const float2* rrow = ep.rope ? ep.rope + (int64_t)(m % ep.rope_rows) * 64 : nullptr;
  bf16* dst = ep.C + (int64_t)m * ep.ldc + n_head;
#pragma unroll 1
  for (int c = 0; c < 4; ++c) {
    uint32_t r[32];
    tmem_ld32(t_head + (uint32_t)(c * 32), r);
    if (!row_ok) continue;
    float v[32];
    const uint4* bp = reinterpret_cast<const uint4*>(ep.bias + n_head + c * 32);
    const uint4* sp = reinterpret_cast<const uint4*>(sc + c * 32);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint4 u = ep.bias ? __ldg(bp + q) : make_uint4(0, 0, 0, 0);
      uint4 w = sc ? __ldg(sp + q) : make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
      const float b8[8] = {bf16_lo(u.x), bf16_hi(u.x), bf16_lo(u.y), bf16_hi(u.y),
                           bf16_lo(u.z), bf16_hi(u.z), bf16_lo(u.w), bf16_hi(u.w)};
      const float s8[8] = {bf16_lo(w.x), bf16_hi(w.x), bf16_lo(w.y), bf16_hi(w.y),
                           bf16_lo(w.z), bf16_hi(w.z), bf16_lo(w.w), bf16_hi(w.w)};
#pragma unroll
      for (int j = 0; j < 8; ++j) v[8 * q + j] = (__uint_as_float(r[8 * q + j]) + b8[j]) * rs * s8[j];
    }
    if (rrow != nullptr) {
      const float4* tp = reinterpret_cast<const float4*>(rrow + c * 16);
#pragma unroll
      for (int p2 = 0; p2 < 8; ++p2) {
        const float4 cs = __ldg(tp + p2);  // pairs 2*p2, 2*p2+1 of this chunk
        const float a0 = v[4 * p2], a1 = v[4 * p2 + 1], b0 = v[4 * p2 + 2], b1 = v[4 * p2 + 3];
        v[4 * p2] = a0 * cs.x - a1 * cs.y;
        v[4 * p2 + 1] = a0 * cs.y + a1 * cs.x;
        v[4 * p2 + 2] = b0 * cs.z - b1 * cs.w;
        v[4 * p2 + 3] = b0 * cs.w + b1 * cs.z;
      }
    }
    uint4* dp = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint4 w;
      w.x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
      w.y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
      w.z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
      w.w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
      dp[q] = w;
    }
  }
}

template <int EPI>
__device__ __forceinline__ void epilogue_chunk(const uint32_t (&r)[32], int m, int n0, const Epi& ep) {
  float v[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
  if (EPI != DIT_EPI_NONE && ep.bias != nullptr) {
    const uint4* bp = reinterpret_cast<const uint4*>(ep.bias + n0);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint4 u = __ldg(bp + q);
      v[8 * q + 0] += bf16_lo(u.x); v[8 * q + 1] += bf16_hi(u.x);
      v[8 * q + 2] += bf16_lo(u.y); v[8 * q + 3] += bf16_hi(u.y);
      v[8 * q + 4] += bf16_lo(u.z); v[8 * q + 5] += bf16_hi(u.z);
      v[8 * q + 6] += bf16_lo(u.w); v[8 * q + 7] += bf16_hi(u.w);
    }
  }
  if (EPI == DIT_EPI_BIAS_GELU_COLS) {
    if (n0 >= ep.gelu_col_begin) {
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = gelu_tanh(v[j]);
    }
  }
  if (EPI == DIT_EPI_BIAS_GATED_RESIDUAL) {
    // gate == nullptr: plain residual add (gate 1)
    const int b = m / ep.rows_per_batch;
    const float4* gp = reinterpret_cast<const float4*>(ep.gate + b * ep.gate_stride + n0);
    const uint4* rp = reinterpret_cast<const uint4*>(ep.resid + (int64_t)m * ep.ldr + n0);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint4 u = rp[q];
      float4 g0 = make_float4(1.f, 1.f, 1.f, 1.f), g1 = g0;
      if (ep.gate != nullptr) {
        g0 = __ldg(gp + 2 * q);
        g1 = __ldg(gp + 2 * q + 1);
      }
      v[8 * q + 0] = fmaf(g0.x, v[8 * q + 0], bf16_lo(u.x));
      v[8 * q + 1] = fmaf(g0.y, v[8 * q + 1], bf16_hi(u.x));
      v[8 * q + 2] = fmaf(g0.z, v[8 * q + 2], bf16_lo(u.y));
      v[8 * q + 3] = fmaf(g0.w, v[8 * q + 3], bf16_hi(u.y));
      v[8 * q + 4] = fmaf(g1.x, v[8 * q + 4], bf16_lo(u.z));
      v[8 * q + 5] = fmaf(g1.y, v[8 * q + 5], bf16_hi(u.z));
      v[8 * q + 6] = fmaf(g1.z, v[8 * q + 6], bf16_lo(u.w));
      v[8 * q + 7] = fmaf(g1.w, v[8 * q + 7], bf16_hi(u.w));
    }
  }
  bf16* dst;
  if (ep.C2 != nullptr && n0 >= ep.split_col)
    dst = ep.C2 + (int64_t)m * ep.ldc2 + (n0 - ep.split_col);
  else
    dst = ep.C + (int64_t)m * ep.ldc + n0;
  uint4* dp = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 w;
    w.x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
    w.y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
    w.z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
    w.w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
    dp[q] = w;
  }
}

template <int EPI>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int M, int N,
                int K, Epi ep, uint64_t wait_limit) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;   // [2]
  uint64_t* tempty = tfull + 2;       // [2]
  uint64_t* drain = tempty + 2;       // [1] abort-path MMA drain
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 4);  // one arrival per epilogue warp
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int num_m = (M + BM - 1) / BM;
  const int num_n = (N + BN - 1) / BN;
  const int num_tiles = num_m * num_n;
  const int num_kb = (K + BK - 1) / BK;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      int stage = 0;
      uint32_t phase = 0;
      // per stage: parity of the most recent fill we issued (for the abort drain)
      uint32_t issued_mask = 0, issued_parity = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int tm = tile % num_m, tn = tile / num_m;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, wait_limit, abort_flag, SITE_GEMM_PRODUCER)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], STAGE_BYTES);
          tma_load_2d(sA + stage * A_BYTES, &tmA, &full[stage], kb * BK, tm * BM);
          tma_load_2d(sB + stage * B_BYTES, &tmB, &full[stage], kb * BK, tn * BN);
          issued_mask |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok) {
        // Let every copy we started land before the CTA exits.
        for (int s = 0; s < STAGES; ++s)
          if (issued_mask & (1u << s))
            (void)mbar_wait(&full[s], (issued_parity >> s) & 1u, wait_limit, nullptr, SITE_GEMM_DRAIN);
      }
    }
  } else if (warp == 1) {
    {
      // ---------------- MMA issuer: the whole warp runs the loop, one
      // elected lane issues each tcgen05 instruction ----------------
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      bool issued_any = false;
      const uint64_t dA = sdesc_sw128(smem_u32(sA), 16, 1024);
      const uint64_t dB = sdesc_sw128(smem_u32(sB), 16, 1024);
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        if (!__all_sync(0xffffffffu, mbar_wait(&tempty[acc], acc_phase ^ 1, wait_limit, abort_flag, SITE_GEMM_MMA))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!__all_sync(0xffffffffu, mbar_wait(&full[stage], phase, wait_limit, abort_flag, SITE_GEMM_MMA))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t a0 = dA + (uint64_t)((stage * A_BYTES) >> 4);
          const uint64_t b0 = dB + (uint64_t)((stage * B_BYTES) >> 4);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            umma_ss_elect(d_tmem, a0 + (uint64_t)(k * 2), b0 + (uint64_t)(k * 2), IDESC, (kb | k) != 0 ? 1u : 0u);
          issued_any = true;
          umma_commit_elect(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        umma_commit_elect(&tfull[acc]);
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1;
        }
      }
      if (!ok && issued_any) {
        // Make sure no MMA still writes TMEM when it is released.
        umma_commit_elect(drain);
        (void)mbar_wait(drain, 0, wait_limit, nullptr, SITE_GEMM_DRAIN);
      }
    }
  } else {
    // ---------------- epilogue warps 2..5 ----------------
    const int quad = warp & 3;  // TMEM lanes quad*32 .. quad*32+31
    const int row_in_tile = quad * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      const int tm = tile % num_m, tn = tile / num_m;
      bool ok = mbar_wait(&tfull[acc], acc_phase, wait_limit, abort_flag, SITE_GEMM_EPILOGUE);
      if (!__all_sync(0xffffffffu, ok)) break;  // keep the warp converged for tcgen05.ld
      tc_fence_after();
      const int m = tm * BM + row_in_tile;
      const uint32_t t_row = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * BN);
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        const int n0 = tn * BN + c * 32;
        if (n0 >= N) break;  // warp-uniform
        if (EPI != DIT_EPI_BIAS_GATED_RESIDUAL && n0 < ep.qk_cols) {
          // a whole 128-column q/k head (heads are 128-aligned, tiles 256-aligned)
          epilogue_qk_head(t_row + (uint32_t)(c * 32), m, n0, ep, m < M);
          c += 3;
          continue;
        }
        uint32_t r[32];
        tmem_ld32(t_row + (uint32_t)(c * 32), r);
        if (m < M) epilogue_chunk<EPI>(r, m, n0, ep);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, TMEM_COLS);
}

// ---------------------------------------------------------------------------
// Two-CTA variant: a cluster of two CTAs on an SM pair computes a 256 x 256
// tile.  CTA r loads rows [128r, 128r+128) of the A tile and rows
// [128r, 128r+128) of the B tile (half of N) into its own shared memory; the
// leader (r = 0) issues tcgen05.mma.cta_group::2 (M=256, N=256, K=16), which
// reads both halves of each operand and writes each CTA's 128 x 256 part of
// the accumulator into that CTA's TMEM.  Per SM this halves the B-operand
// traffic of the one-CTA tile, and with 32 KB stages six fit in shared memory.
// No TMA multicast: each CTA fetches its own halves.
//   - full[s] (leader): one arrival (the leader's expect_tx for both CTAs'
//     bytes) plus the transaction bytes of both CTAs' loads;
//   - empty[s] (both): committed by the leader's MMA thread to both CTAs;
//   - tfull[a] (both): committed to both CTAs after the last K block;
//   - tempty[a] (leader): 8 arrivals, 4 epilogue warps in each CTA.
// ---------------------------------------------------------------------------
namespace pair {

// Tile order.  M-fastest (n_fastest = 0): the clusters running together share
// B panels, and every wave re-reads the whole A operand, so A should be the
// smaller operand (it then stays in L2 from wave to wave).  N-fastest: the
// other way round, for GEMMs whose A is larger than their weight (the output
// projections: A = [S, D+M], W = [D, D+M]).
__device__ __forceinline__ void tile_coords(int tile, int num_m, int num_n, int n_fastest, int& tm, int& tn) {
  if (n_fastest) {
    tm = tile / num_n;
    tn = tile - tm * num_n;
  } else {
    tn = tile / num_m;
    tm = tile - tn * num_m;
  }
}

constexpr int BM = 256;      // rows per cluster tile
constexpr int BM_CTA = 128;  // rows per CTA
constexpr int BN = 256;
constexpr int BN_CTA = 128;  // B rows loaded per CTA
constexpr int BK = 64;
constexpr int STAGES = 6;
constexpr int A_BYTES = BM_CTA * BK * 2;
constexpr int B_BYTES = BN_CTA * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int NUM_THREADS = 192;
constexpr uint32_t TMEM_COLS = 512;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 256 + 1024;
constexpr uint32_t IDESC = idesc_bf16(BM, BN, 0, 0);

// One GEMM of a launch: its operands' tensor maps, epilogue, shape and tile
// order.  A launch runs one job or a group of two with the same K and
// epilogue kind (the double-stream block's text and image projections): the
// tiles of job 1 follow those of job 0 in one persistent schedule, so a job
// with few tiles fills the SMs the other leaves idle.
struct PairJob {
  CUtensorMap tmA, tmB;
  Epi ep;
  int M, N;
  int n_fastest;
};
struct PairGroup {
  PairJob job[2];
  int count;  // 1 or 2
};

// tile index of the launch -> job and tile coordinates
__device__ __forceinline__ int group_tile(const PairGroup& G, int tiles0, int tile, int& tm, int& tn) {
  const int g = (G.count > 1 && tile >= tiles0) ? 1 : 0;
  const PairJob& J = G.job[g];
  tile_coords(g ? tile - tiles0 : tile, (J.M + BM - 1) / BM, (J.N + BN - 1) / BN, J.n_fastest, tm, tn);
  return g;
}

// Work items of the persistent schedule.  The tiles of the complete waves
// run whole.  When the last, partial wave holds at most half as many tiles as
// there are clusters, each of its tiles runs as two items of 128 columns
// (N = 128 MMAs) on two clusters, so that wave takes half a tile's time:
// the fused QKV|MLP-in GEMM of the single-stream block at S = 4608 has 1512
// tiles for 74 SM pairs, 20 whole waves and 32 tiles left.
constexpr int BN_HALF = 128;
constexpr uint32_t IDESC_HALF = idesc_bf16(BM, BN_HALF, 0, 0);

struct TailPlan {
  int full;   // tiles that run whole (complete waves, or every tile without a split)
  int items;  // work items in all
};
__device__ __forceinline__ TailPlan tail_plan(int num_tiles, int n_clusters) {
  const int full = num_tiles / n_clusters * n_clusters;
  const int rem = num_tiles - full;
  if (rem > 0 && 2 * rem <= n_clusters) return TailPlan{full, full + 2 * rem};
  return TailPlan{num_tiles, num_tiles};
}
// item -> tile and column half (-1: the whole tile)
__device__ __forceinline__ int item_tile(const TailPlan& P, int item, int& half) {
  if (item < P.full) {
    half = -1;
    return item;
  }
  half = (item - P.full) & 1;
  return P.full + ((item - P.full) >> 1);
}

template <int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NUM_THREADS, 1)
    gemm_pair_kernel(const __grid_constant__ PairGroup G, int K, uint64_t wait_limit) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;  // [2]
  uint64_t* tempty = tfull + 2;      // [2]
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 8);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    for (int g = 0; g < G.count; ++g) {
      tma_prefetch_desc(&G.job[g].tmA);
      tma_prefetch_desc(&G.job[g].tmB);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // barrier inits and TMEM allocation visible to both CTAs
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  griddep_wait();  // the prologue above overlaps the previous kernel; everything below follows it
  griddep_launch_dependents();

  const int tiles0 = ((G.job[0].M + BM - 1) / BM) * ((G.job[0].N + BN - 1) / BN);
  const int num_tiles =
      tiles0 + (G.count > 1 ? ((G.job[1].M + BM - 1) / BM) * ((G.job[1].N + BN - 1) / BN) : 0);
  const int num_kb = (K + BK - 1) / BK;
  const int cluster_id = blockIdx.x >> 1;
  const int n_clusters = gridDim.x >> 1;
  const TailPlan plan = tail_plan(num_tiles, n_clusters);

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (both CTAs) ----------------
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_parity = 0;
      bool ok = true;
      int wave = 0;  // this cluster's tile count so far: the same for every cluster of a wave
      const uint64_t b_policy = l2_policy_evict_last();
      for (int item = cluster_id; item < plan.items && ok; item += n_clusters, ++wave) {
        int tm, tn, half;
        const PairJob& J = G.job[group_tile(G, tiles0, item_tile(plan, item, half), tm, tn)];
        // B rows of this CTA: its half of the tile's 256 columns, or of the
        // 128 columns of a half item (the box still loads 128 rows; the MMA
        // reads the first 64)
        const int b_row = tn * BN + (half < 0 ? (int)rank * BN_CTA : half * BN_HALF + (int)rank * (BN_HALF / 2));
        const bool keep_b = J.n_fastest && J.ep.w_keep != nullptr;
        // N-fastest: every other wave walks K backwards, so that it starts on the
        // K range whose weight panels the previous wave touched last (still in L2)
        const bool back = J.n_fastest && (wave & 1);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, wait_limit, abort_flag, SITE_GEMM2_PRODUCER)) {
            ok = false;
            break;
          }
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * STAGE_BYTES);
          const uint32_t leader_full = mapa_shared(smem_u32(&full[stage]), 0);
          const int kx = (back ? num_kb - 1 - kb : kb) * BK;
          tma_load_2d_pair(sA + stage * A_BYTES, &J.tmA, leader_full, kx, tm * BM + (int)rank * BM_CTA);
          if (keep_b)
            tma_load_2d_pair_hint(sB + stage * B_BYTES, &J.tmB, leader_full, kx, b_row, b_policy);
          else
            tma_load_2d_pair(sB + stage * B_BYTES, &J.tmB, leader_full, kx, b_row);
          issued_mask |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok && rank == 0) {
        for (int s = 0; s < STAGES; ++s)
          if (issued_mask & (1u << s))
            (void)mbar_wait(&full[s], (issued_parity >> s) & 1u, wait_limit, nullptr, SITE_GEMM2_DRAIN);
      }
    }
  } else if (warp == 1) {
    if (rank == 0) {
      // ---------------- MMA issuer (leader CTA): the whole warp runs the
      // loop, one elected lane issues each tcgen05 instruction ----------------
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      bool issued_any = false;
      // descriptor of stage 0's A and B tiles; a stage or a 16-deep slice adds (byte offset >> 4)
      const uint64_t dA = sdesc_sw128(smem_u32(sA), 16, 1024);
      const uint64_t dB = sdesc_sw128(smem_u32(sB), 16, 1024);
      for (int item = cluster_id; item < plan.items && ok; item += n_clusters) {
        int half;
        (void)item_tile(plan, item, half);
        const uint32_t idesc = half < 0 ? IDESC : IDESC_HALF;
        if (!__all_sync(0xffffffffu, mbar_wait(&tempty[acc], acc_phase ^ 1, wait_limit, abort_flag, SITE_GEMM2_MMA))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!__all_sync(0xffffffffu, mbar_wait(&full[stage], phase, wait_limit, abort_flag, SITE_GEMM2_MMA))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t a0 = dA + (uint64_t)((stage * A_BYTES) >> 4);
          const uint64_t b0 = dB + (uint64_t)((stage * B_BYTES) >> 4);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            umma_ss_pair_elect(d_tmem, a0 + (uint64_t)(k * 2), b0 + (uint64_t)(k * 2), idesc, (kb | k) != 0 ? 1u : 0u);
          issued_any = true;
          umma_commit_pair_elect(&empty[stage], 0x3);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        umma_commit_pair_elect(&tfull[acc], 0x3);
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1;
        }
      }
      if (!ok && issued_any) {
        umma_commit_elect(drain);
        (void)mbar_wait(drain, 0, wait_limit, nullptr, SITE_GEMM2_DRAIN);
      }
    }
  } else {
    // ---------------- epilogue warps 2..5 (both CTAs) ----------------
    const int quad = warp & 3;
    const int row_in_tile = (int)rank * BM_CTA + quad * 32 + lane;
    const uint32_t leader_tempty0 = mapa_shared(smem_u32(&tempty[0]), 0);
    const uint32_t leader_tempty1 = mapa_shared(smem_u32(&tempty[1]), 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int item = cluster_id; item < plan.items; item += n_clusters) {
      int tm, tn, half;
      const PairJob& J = G.job[group_tile(G, tiles0, item_tile(plan, item, half), tm, tn)];
      const int col0 = tn * BN + (half < 0 ? 0 : half * BN_HALF);  // first output column of the item
      const int chunks = (half < 0 ? BN : BN_HALF) / 32;
      const Epi& ep = J.ep;
      const int M = J.M, N = J.N;
      bool ok = mbar_wait(&tfull[acc], acc_phase, wait_limit, abort_flag, SITE_GEMM2_EPILOGUE);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const int m = tm * BM + row_in_tile;
      const uint32_t t_row = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * BN);
#pragma unroll 1
      for (int c = 0; c < chunks; ++c) {
        const int n0 = col0 + c * 32;
        if (n0 >= N) break;  // warp-uniform
        if (EPI != DIT_EPI_BIAS_GATED_RESIDUAL && n0 < ep.qk_cols) {
          epilogue_qk_head(t_row + (uint32_t)(c * 32), m, n0, ep, m < M);
          c += 3;
          continue;
        }
        uint32_t r[32];
        tmem_ld32(t_row + (uint32_t)(c * 32), r);
        if (m < M) epilogue_chunk<EPI>(r, m, n0, ep);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc ? leader_tempty1 : leader_tempty0);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
  }

  tc_fence_before();
  cluster_sync_all();  // no CTA leaves while its peer may still touch its memory
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, TMEM_COLS);
  for (int g = 0; g < G.count; ++g) {
    const PairJob& J = G.job[g];
    if (J.n_fastest && J.ep.w_keep != nullptr) {
      // this CTA's share of the kept weight back to normal L2 priority
      const int64_t lines = J.ep.w_keep_bytes >> 7;
      for (int64_t i = (int64_t)blockIdx.x * NUM_THREADS + threadIdx.x; i < lines;
           i += (int64_t)gridDim.x * NUM_THREADS)
        l2_priority_normal(J.ep.w_keep + (i << 7));
    }
  }
}

}  // namespace pair
}  // namespace gemm
}  // namespace dit

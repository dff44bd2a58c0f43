// HBM-bound kernels of the block: adaLN modulation (vector x weight), fused
// LayerNorm + adaLN modulate, fused QK RMSNorm + RoPE, the RoPE table, and the
// small loop kernels (timestep embedding, patchify, Euler update).
//
// Page: "compile_graph" (chenyy20.com), §1.1 — LayerNorm, GELU and
// (1+scale)*x+shift are memory-bound; each separate kernel is a full HBM round
// trip, so each of these makes exactly one coalesced pass over its rows.
#pragma once

#include "common.cuh"

namespace dit {

// ---------------------------------------------------------------------------
// Block-wide sum over blockDim.x threads (blockDim.x a multiple of 32).
// ---------------------------------------------------------------------------
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}


// ---------------------------------------------------------------------------
// LayerNorm + modulate, persistent row stream: a CTA of D/8 threads walks rows
// blockIdx.x, blockIdx.x + gridDim.x, ...; thread t always owns columns
// [8t, 8t+8), so its 8 shift and 8 scale values stay in registers for every
// row of the batch, and it loads the next row's 16 bytes before reducing the
// current one.  Per row the only memory traffic is one 16-byte load and one
// 16-byte store per thread.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) modulate_norm_stream_kernel(const bf16* __restrict__ x, int64_t ldx,
                                                                    const float* __restrict__ shift,
                                                                    const float* __restrict__ scale,
                                                                    int64_t mod_stride, bf16* __restrict__ y,
                                                                    int64_t ldy, int64_t rows, int S, int D,
                                                                    float eps) {
  __shared__ float red[2][32];
  const int c0 = threadIdx.x * 8;
  const bool active = c0 < D;
  const float invD = 1.0f / (float)D;
  int64_t r = blockIdx.x;
  uint4 cur = make_uint4(0, 0, 0, 0);
  if (active && r < rows) cur = __ldcs(reinterpret_cast<const uint4*>(x + r * ldx + c0));
  int cur_b = -1;
  float sh[8], sc1[8];
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31, nw = blockDim.x >> 5;
  int par = 0;
  for (; r < rows; r += gridDim.x) {
    const int64_t rn = r + gridDim.x;
    uint4 nxt = make_uint4(0, 0, 0, 0);
    if (active && rn < rows) nxt = __ldcs(reinterpret_cast<const uint4*>(x + rn * ldx + c0));
    const int b = (int)(r / S);
    if (b != cur_b) {  // new batch row: refresh this thread's modulation (uniform across the CTA)
      cur_b = b;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        sh[i] = 0.0f;
        sc1[i] = 1.0f;
      }
      if (active && shift != nullptr) {
        const float4* ps = reinterpret_cast<const float4*>(shift + b * mod_stride + c0);
        const float4* pc = reinterpret_cast<const float4*>(scale + b * mod_stride + c0);
        const float4 a0 = __ldg(ps), a1 = __ldg(ps + 1), b0 = __ldg(pc), b1 = __ldg(pc + 1);
        sh[0] = a0.x; sh[1] = a0.y; sh[2] = a0.z; sh[3] = a0.w; sh[4] = a1.x; sh[5] = a1.y; sh[6] = a1.z; sh[7] = a1.w;
        sc1[0] = 1.f + b0.x; sc1[1] = 1.f + b0.y; sc1[2] = 1.f + b0.z; sc1[3] = 1.f + b0.w;
        sc1[4] = 1.f + b1.x; sc1[5] = 1.f + b1.y; sc1[6] = 1.f + b1.z; sc1[7] = 1.f + b1.w;
      }
    }
    const float v[8] = {bf16_lo(cur.x), bf16_hi(cur.x), bf16_lo(cur.y), bf16_hi(cur.y),
                        bf16_lo(cur.z), bf16_hi(cur.z), bf16_lo(cur.w), bf16_hi(cur.w)};
    // mean (inactive threads hold zeros)
    float t = ((v[0] + v[1]) + (v[2] + v[3])) + ((v[4] + v[5]) + (v[6] + v[7]));
    t = warp_sum(t);
    if (l == 0) red[par][w] = t;
    __syncthreads();
    float tot = (l < nw) ? red[par][l] : 0.0f;
    const float mean = warp_sum(tot) * invD;
    // centred second moment from the same registers
    float q = 0.0f;
    if (active) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float d = v[i] - mean;
        q = fmaf(d, d, q);
      }
    }
    q = warp_sum(q);
    par ^= 1;  // the other buffer: no thread can still be reading it
    if (l == 0) red[par][w] = q;
    __syncthreads();
    tot = (l < nw) ? red[par][l] : 0.0f;
    const float rstd = rsqrtf(warp_sum(tot) * invD + eps);
    par ^= 1;
    if (active) {
      uint4 o;
      o.x = pack_bf16x2(fmaf(sc1[0], (v[0] - mean) * rstd, sh[0]), fmaf(sc1[1], (v[1] - mean) * rstd, sh[1]));
      o.y = pack_bf16x2(fmaf(sc1[2], (v[2] - mean) * rstd, sh[2]), fmaf(sc1[3], (v[3] - mean) * rstd, sh[3]));
      o.z = pack_bf16x2(fmaf(sc1[4], (v[4] - mean) * rstd, sh[4]), fmaf(sc1[5], (v[5] - mean) * rstd, sh[5]));
      o.w = pack_bf16x2(fmaf(sc1[6], (v[6] - mean) * rstd, sh[6]), fmaf(sc1[7], (v[7] - mean) * rstd, sh[7]));
      *reinterpret_cast<uint4*>(y + r * ldy + c0) = o;
    }
    cur = nxt;
  }
}

// ---------------------------------------------------------------------------
// LayerNorm + modulate, persistent row ring: CTA (j, b) owns the rows j,
// j + gridDim.x, ... of batch row b.  Thread 0 keeps R of them in flight as
// whole-row bulk copies into a ring of R shared-memory stages, so the bytes
// an SM has requested from HBM do not run out while the CTA reduces and
// writes a row; waits poll the barrier without suspending.  Thread t owns the
// 16-byte chunks t, t + T, ... of every row (T = D / (8 NC)), so its
// (1 + scale) and shift values are read once and stay in registers.
// Statistics in one pass over data shifted by the row's first element K:
// d = x - K, mean = K + sum(d) / D, variance = sum(d^2) / D - (sum(d) / D)^2
// (the shifted-data algorithm).  The cancellation in the variance is bounded
// by (K - mean)^2 / variance <= D, so its relative error stays below about
// D * 2^-24 (2e-4 at D = 3072) for any row, and a row of equal values gets
// d = 0, variance 0 and output exactly the shift.  One reduction per row
// (both sums share the shuffles) and one barrier, which also tells thread 0
// that every thread has read the stage; it then refills it with the row R
// ahead.  Packed fp32 pairs throughout: at D = 3072 the per-row chain of
// dependent steps costs about as much as the row's HBM traffic.
// ---------------------------------------------------------------------------
constexpr int kNormRingMaxStages = 8;

template <int NC>
__global__ void __launch_bounds__(256) modulate_norm_ring_kernel(const bf16* __restrict__ x, int64_t ldx,
                                                                 const float* __restrict__ shift,
                                                                 const float* __restrict__ scale,
                                                                 int64_t mod_stride, bf16* __restrict__ y,
                                                                 int64_t ldy, int S, int D, float eps, int R,
                                                                 uint64_t wait_limit) {
  constexpr int H = 4 * NC;  // packed pairs per thread and row
  extern __shared__ __align__(128) uint8_t ring[];  // R stages of one row (D bf16) each
  __shared__ __align__(8) uint64_t full[kNormRingMaxStages];
  __shared__ float2 red[2][8];  // per warp (sum d, sum d^2), two rows apart
  const int T = blockDim.x;
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31, nw = T >> 5;
  const int b = blockIdx.y;
  const int G = (int)gridDim.x;
  const int n = (S - 1 - (int)blockIdx.x) / G + 1;  // rows of this CTA (gridDim.x <= S)
  const uint32_t row_bytes = (uint32_t)D * 2u;
  const float inv_d = 1.0f / (float)D;
  if (threadIdx.x == 0) {
    for (int s = 0; s < R; ++s) mbar_init(&full[s], 1);
    fence_mbar_init();
  }
  __syncthreads();
  griddep_wait();
  griddep_launch_dependents();
  const bf16* xrow0 = x + ((int64_t)b * S + blockIdx.x) * ldx;  // the CTA's first row
  const int64_t src_step = (int64_t)G * ldx;
  if (threadIdx.x == 0) {
    for (int k = 0; k < R && k < n; ++k) {
      mbar_arrive_expect_tx(&full[k], row_bytes);
      bulk_load(ring + (size_t)k * row_bytes, xrow0 + k * src_step, row_bytes, &full[k]);
    }
  }
  uint64_t sc1[H], sh[H];
#pragma unroll
  for (int c = 0; c < NC; ++c) {
    const int col = (c * T + threadIdx.x) * 8;
    if (shift != nullptr) {
      const float4* ps = reinterpret_cast<const float4*>(shift + b * mod_stride + col);
      const float4* pc = reinterpret_cast<const float4*>(scale + b * mod_stride + col);
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const float4 a = __ldg(ps + q), sc = __ldg(pc + q);
        sh[c * 4 + q * 2] = f2_pack(a.x, a.y);
        sh[c * 4 + q * 2 + 1] = f2_pack(a.z, a.w);
        sc1[c * 4 + q * 2] = f2_pack(1.f + sc.x, 1.f + sc.y);
        sc1[c * 4 + q * 2 + 1] = f2_pack(1.f + sc.z, 1.f + sc.w);
      }
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        sh[c * 4 + q] = 0ull;
        sc1[c * 4 + q] = f2_pack(1.f, 1.f);
      }
    }
  }
  uint4* yr = reinterpret_cast<uint4*>(y + ((int64_t)b * S + blockIdx.x) * ldy) + threadIdx.x;
  const int64_t y_step = (int64_t)G * ldy / 8;  // in 16-byte chunks
  int i = 0;
  for (; i < n; ++i, yr += y_step) {
    const int s = i % R;
    const bool ok = mbar_wait_poll(&full[s], (uint32_t)(i / R) & 1u, wait_limit, SITE_NORM_RING);
    const uint8_t* stage = ring + (size_t)s * row_bytes;
    const uint4* xr = reinterpret_cast<const uint4*>(stage) + threadIdx.x;
    const float k0 = bf16_lo(*reinterpret_cast<const uint32_t*>(stage));  // the shift K: the row's first value
    const uint64_t negk = f2_pack(-k0, -k0);
    uint4 u4[NC];
#pragma unroll
    for (int c = 0; c < NC; ++c) u4[c] = xr[c * T];
    uint64_t d[H];
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      const uint32_t u[4] = {u4[c].x, u4[c].y, u4[c].z, u4[c].w};
#pragma unroll
      for (int q = 0; q < 4; ++q) d[c * 4 + q] = f2_add(f2_pack(bf16_lo(u[q]), bf16_hi(u[q])), negk);
    }
    uint64_t s1 = d[0], s2 = f2_mul(d[0], d[0]);
#pragma unroll
    for (int k = 1; k < H; ++k) {
      s1 = f2_add(s1, d[k]);
      s2 = f2_fma(d[k], d[k], s2);
    }
    float a1 = f2_lo(s1) + f2_hi(s1), a2 = f2_lo(s2) + f2_hi(s2);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      a1 += __shfl_xor_sync(0xffffffffu, a1, o);
      a2 += __shfl_xor_sync(0xffffffffu, a2, o);
    }
    if (l == 0) red[i & 1][w] = make_float2(a1, a2);
    // every thread has read stage s and published its warp's sums; a wait
    // that ran out in any thread ends the CTA's loop in all of them
    if (__syncthreads_or(!ok)) break;
    if (threadIdx.x == 0 && i + R < n) {  // refill stage s with the row R ahead
      mbar_arrive_expect_tx(&full[s], row_bytes);
      bulk_load(ring + (size_t)s * row_bytes, xrow0 + (int64_t)(i + R) * src_step, row_bytes, &full[s]);
    }
    float t1 = 0.0f, t2 = 0.0f;
    for (int k = 0; k < nw; ++k) {
      const float2 r = red[i & 1][k];
      t1 += r.x;
      t2 += r.y;
    }
    const float md = t1 * inv_d;  // mean of d
    const float rstd = rsqrtf(fmaxf(fmaf(-md, md, t2 * inv_d), 0.0f) + eps);
    // y = (d - mean of d) rstd (1 + scale) + shift
    const uint64_t rstd2 = f2_pack(rstd, rstd);
    const uint64_t nmr2 = f2_pack(-md * rstd, -md * rstd);
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      uint32_t pk[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint64_t o = f2_fma(f2_fma(d[c * 4 + q], rstd2, nmr2), sc1[c * 4 + q], sh[c * 4 + q]);
        pk[q] = pack_bf16x2(f2_lo(o), f2_hi(o));
      }
      yr[c * T] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
  }
  if (i < n && threadIdx.x == 0) {
    // a wait ran out at row i: let the copies that may still be in flight
    // (rows i .. i + R - 1) land before the CTA's shared memory is released
    for (int j = i; j < i + R && j < n; ++j)
      (void)mbar_wait_poll(&full[j % R], (uint32_t)(j / R) & 1u, wait_limit, SITE_NORM_RING);
  }
}

// ---------------------------------------------------------------------------
// Vector x weight rows (adaLN modulation, the timestep MLP), batch NB <= 2,
// K = 256 KC: one warp per output row, lane l reading the 16-byte chunks
// l, l + 32, ... of the row with streaming loads, the (mapped) input vectors
// in shared memory as fp32.  They are stored lane-interleaved: the 8 values
// lane l needs for chunk c sit as float4 [c][l] (first 4) and [c][32 + l]
// (last 4), so a warp's shared-memory reads are contiguous (no bank
// conflicts).  A warp issues the loads of its next row as soon as a row is
// reduced, and keeps two rows in flight while the registers allow it; rows
// are dealt to the warps of a persistent grid round robin.  RowFn(n) gives
// row n's weight pointer, bias and output slot, so the same loop serves one
// matrix and a list of matrices that share the input (every block's
// modulation of a step).
// ---------------------------------------------------------------------------
struct VecRow {
  const uint4* w;
  const bf16* bias;
  int64_t local;  // index of the row within its matrix
  int mat;        // which matrix (0 for a single matrix)
};

template <int KC>
__device__ __forceinline__ void vr_load(uint4 (&u)[KC], float& bv, const VecRow& rw, bool on, int lane) {
#pragma unroll
  for (int c = 0; c < KC; ++c) u[c] = on ? __ldcs(rw.w + c * 32 + lane) : make_uint4(0, 0, 0, 0);
  bv = (on && lane == 0 && rw.bias != nullptr) ? __bfloat162float(rw.bias[rw.local]) : 0.0f;
}

// dot products of the row held in u with input vector b (interleaved layout, 64 float4 per chunk)
template <int KC>
__device__ __forceinline__ float vr_dot(const uint4 (&u)[KC], const float4* __restrict__ xs, int lane) {
  float a0 = 0.f, a1 = 0.f;
#pragma unroll
  for (int c = 0; c < KC; ++c) {
    const float4 x0 = xs[c * 64 + lane], x1 = xs[c * 64 + 32 + lane];
    a0 = fmaf(bf16_lo(u[c].x), x0.x, a0); a1 = fmaf(bf16_hi(u[c].x), x0.y, a1);
    a0 = fmaf(bf16_lo(u[c].y), x0.z, a0); a1 = fmaf(bf16_hi(u[c].y), x0.w, a1);
    a0 = fmaf(bf16_lo(u[c].z), x1.x, a0); a1 = fmaf(bf16_hi(u[c].z), x1.y, a1);
    a0 = fmaf(bf16_lo(u[c].w), x1.z, a0); a1 = fmaf(bf16_hi(u[c].w), x1.w, a1);
  }
  return warp_sum(a0 + a1);
}

template <int KC, int NB, typename RowFn, typename OutFn>
__device__ __forceinline__ void vec_rows_loop(const bf16* __restrict__ x, int64_t ldx, int K, int flags, int64_t N,
                                              RowFn row_of, OutFn store) {
  constexpr bool TWO = KC * NB <= 6;  // two rows in flight per warp while the registers allow it
  griddep_wait();
  griddep_launch_dependents();
  extern __shared__ float4 xs4[];  // NB mapped inputs, K fp32 each, lane-interleaved
  float* xs = reinterpret_cast<float*>(xs4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t nw = (int64_t)gridDim.x * (blockDim.x >> 5);
  const int64_t step = TWO ? 2 * nw : nw;
  int64_t n = (int64_t)blockIdx.x * (blockDim.x >> 5) + warp;
  uint4 ua[KC], ub[TWO ? KC : 1];
  float ba = 0.f, bb = 0.f;
  VecRow ra = row_of(n < N ? n : 0), rb = ra;
  vr_load<KC>(ua, ba, ra, n < N, lane);
  if constexpr (TWO) {
    rb = row_of(n + nw < N ? n + nw : 0);
    vr_load<KC>(ub, bb, rb, n + nw < N, lane);
  }
  for (int i = threadIdx.x; i < NB * K; i += blockDim.x) {
    const int b = i / K, k = i - b * K;
    float z = __bfloat162float(x[b * ldx + k]);
    if (flags & DIT_VEC_SILU_IN) z = silu(z);
    // column k = 8 (32 c + l) + j sits in float4 [c][l] (j < 4) or [c][32 + l] (j >= 4)
    const int c = k >> 8, l = (k >> 3) & 31, j = k & 7;
    xs[b * K + ((c * 64 + (j >> 2) * 32 + l) << 2) + (j & 3)] = z;
  }
  __syncthreads();
  for (; n < N; n += step) {
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      const float da = vr_dot<KC>(ua, xs4 + b * (K / 4), lane) + ba;
      if (lane == 0) store(ra, b, da);
    }
    const int64_t n2 = n + step;
    ra = row_of(n2 < N ? n2 : 0);
    vr_load<KC>(ua, ba, ra, n2 < N, lane);
    if constexpr (TWO) {
      if (n + nw < N) {
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          const float db = vr_dot<KC>(ub, xs4 + b * (K / 4), lane) + bb;
          if (lane == 0) store(rb, b, db);
        }
      }
      const int64_t n3 = n + nw + step;
      rb = row_of(n3 < N ? n3 : 0);
      vr_load<KC>(ub, bb, rb, n3 < N, lane);
    }
  }
}

template <int KC, int NB>
__global__ void __launch_bounds__(512, 1) vec_rows_kernel(const bf16* __restrict__ x, int64_t ldx,
                                                          const bf16* __restrict__ W, int64_t ldw,
                                                          const bf16* __restrict__ bias, void* out, int64_t ldo,
                                                          int64_t N, int K, int flags) {
  vec_rows_loop<KC, NB>(
      x, ldx, K, flags, N,
      [=](int64_t n) { return VecRow{reinterpret_cast<const uint4*>(W + n * ldw), bias, n, 0}; },
      [=](const VecRow& rw, int b, float v) {
        if (flags & DIT_VEC_OUT_BF16)
          reinterpret_cast<bf16*>(out)[b * ldo + rw.local] = __float2bfloat16_rn(v);
        else
          reinterpret_cast<float*>(out)[b * ldo + rw.local] = v;
      });
}

// ---------------------------------------------------------------------------
// adaLN / vector x weight, batch 1, with the weight rows in flight through a
// warp-private shared-memory ring of P row slots.  Lane l copies its KC
// 16-byte chunks (columns 8(l + 32j) .. +8) of the warp's next rows into the
// ring with cp.async, P - 1 rows ahead, and reads back exactly what it copied
// (no barrier); the input vector is held in registers in the same column
// order.  One warp per output feature, features dealt round-robin; 4 warps
// per CTA.
// ---------------------------------------------------------------------------
constexpr int kVecPipeWarps = 4;
constexpr int kVecPipeSlots = 4;

template <int KC>
__global__ void __launch_bounds__(128) vec_linear_pipe_kernel(const bf16* __restrict__ x,
                                                              const bf16* __restrict__ W, int64_t ldw,
                                                              const bf16* __restrict__ bias, void* out, int N,
                                                              int K, int flags) {
  constexpr int P = kVecPipeSlots;
  extern __shared__ __align__(16) uint4 wring[];  // [warps][P][K / 8], then the mapped input (K fp32)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row_chunks = K / 8;
  uint4* ring = wring + (size_t)warp * P * row_chunks;
  float* xs = reinterpret_cast<float*>(wring + (size_t)kVecPipeWarps * P * row_chunks);
  const int64_t nw = (int64_t)gridDim.x * kVecPipeWarps;
  const int64_t n0 = (int64_t)blockIdx.x * kVecPipeWarps + warp;
#pragma unroll
  for (int k = 0; k < P - 1; ++k) {
    const int64_t nn = n0 + k * nw;
    if (nn < N) {
#pragma unroll
      for (int j = 0; j < KC; ++j)
        cp_async16(&ring[k * row_chunks + lane + 32 * j],
                   reinterpret_cast<const uint4*>(W + nn * ldw) + lane + 32 * j);
    }
    cp_async_commit();
  }
  // the mapped input is computed once per CTA, then each lane keeps its columns in registers
  for (int k = threadIdx.x; k < K; k += blockDim.x) {
    float z = __bfloat162float(x[k]);
    if (flags & DIT_VEC_SILU_IN) z = silu(z);
    xs[k] = z;
  }
  __syncthreads();
  float xv[KC * 8];
#pragma unroll
  for (int j = 0; j < KC; ++j) {
    const float4* p = reinterpret_cast<const float4*>(xs + (lane + 32 * j) * 8);
    const float4 a = p[0], c = p[1];
    xv[j * 8 + 0] = a.x; xv[j * 8 + 1] = a.y; xv[j * 8 + 2] = a.z; xv[j * 8 + 3] = a.w;
    xv[j * 8 + 4] = c.x; xv[j * 8 + 5] = c.y; xv[j * 8 + 6] = c.z; xv[j * 8 + 7] = c.w;
  }
  int slot = 0;
  for (int64_t n = n0; n < N; n += nw) {
    {  // the slot consumed one row ago gets the row P - 1 ahead
      const int64_t nn = n + (int64_t)(P - 1) * nw;
      const int si = (slot == 0 ? P : slot) - 1;
      if (nn < N) {
#pragma unroll
        for (int j = 0; j < KC; ++j)
          cp_async16(&ring[si * row_chunks + lane + 32 * j],
                     reinterpret_cast<const uint4*>(W + nn * ldw) + lane + 32 * j);
      }
      cp_async_commit();
    }
    // the bias load is issued before the wait so that its latency overlaps the copies
    const float bv = bias ? __bfloat162float(bias[n]) : 0.0f;
    cp_async_wait<P - 1>();
    float a0 = 0.f, a1 = 0.f;
#pragma unroll
    for (int j = 0; j < KC; ++j) {
      const uint4 u = ring[slot * row_chunks + lane + 32 * j];
      a0 = fmaf(bf16_lo(u.x), xv[j * 8 + 0], a0); a1 = fmaf(bf16_hi(u.x), xv[j * 8 + 1], a1);
      a0 = fmaf(bf16_lo(u.y), xv[j * 8 + 2], a0); a1 = fmaf(bf16_hi(u.y), xv[j * 8 + 3], a1);
      a0 = fmaf(bf16_lo(u.z), xv[j * 8 + 4], a0); a1 = fmaf(bf16_hi(u.z), xv[j * 8 + 5], a1);
      a0 = fmaf(bf16_lo(u.w), xv[j * 8 + 6], a0); a1 = fmaf(bf16_hi(u.w), xv[j * 8 + 7], a1);
    }
    const float a = warp_sum(a0 + a1) + bv;
    if (lane == 0) {
      if (flags & DIT_VEC_OUT_BF16)
        reinterpret_cast<bf16*>(out)[n] = __float2bfloat16_rn(a);
      else
        reinterpret_cast<float*>(out)[n] = a;
    }
    if (++slot == P) slot = 0;
  }
  cp_async_wait<0>();
}

// ---------------------------------------------------------------------------
// The same contraction over a list of matrices that share one input vector:
// every block's adaLN modulation of a denoising step depends only on that
// step's conditioning vector, so all of them stream in one pass.  Global row
// n belongs to matrix j with row_begin[j] <= n < row_begin[j+1] (binary
// search); out[j][n - row_begin[j]] = W_j[row] . f(x) + bias_j[row], fp32.
// Rows are dealt to warps and streamed exactly as in vec_linear_pipe_kernel
// (same column order, same accumulation), so every output equals that
// kernel's output for the same matrix.  Every matrix has K columns, ldw = K.
// ---------------------------------------------------------------------------
constexpr int kMultiMaxMats = 96;
struct MultiLinear {
  const bf16* W[kMultiMaxMats];
  const bf16* bias[kMultiMaxMats];
  float* out[kMultiMaxMats];
  int row_begin[kMultiMaxMats + 1];
  int n_mats;
  int K;
};

__device__ __forceinline__ int multi_find(const MultiLinear& p, int64_t n) {
  int lo = 0, hi = p.n_mats - 1;  // largest j with row_begin[j] <= n
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.row_begin[mid] <= n) lo = mid; else hi = mid - 1;
  }
  return lo;
}

template <int KC>
__global__ void __launch_bounds__(128) vec_linear_multi_kernel(const bf16* __restrict__ x,
                                                               const __grid_constant__ MultiLinear p, int flags) {
  constexpr int P = kVecPipeSlots;
  extern __shared__ __align__(16) uint4 wring[];  // [warps][P][K / 8], then the mapped input (K fp32)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int K = p.K;
  const int row_chunks = K / 8;
  const int64_t N = p.row_begin[p.n_mats];
  uint4* ring = wring + (size_t)warp * P * row_chunks;
  float* xs = reinterpret_cast<float*>(wring + (size_t)kVecPipeWarps * P * row_chunks);
  const int64_t nw = (int64_t)gridDim.x * kVecPipeWarps;
  const int64_t n0 = (int64_t)blockIdx.x * kVecPipeWarps + warp;
  auto row_ptr = [&](int64_t n) -> const uint4* {
    const int j = multi_find(p, n);
    return reinterpret_cast<const uint4*>(p.W[j] + (n - p.row_begin[j]) * K);
  };
#pragma unroll
  for (int k = 0; k < P - 1; ++k) {
    const int64_t nn = n0 + k * nw;
    if (nn < N) {
      const uint4* src = row_ptr(nn);
#pragma unroll
      for (int j = 0; j < KC; ++j) cp_async16(&ring[k * row_chunks + lane + 32 * j], src + lane + 32 * j);
    }
    cp_async_commit();
  }
  for (int k = threadIdx.x; k < K; k += blockDim.x) {
    float z = __bfloat162float(x[k]);
    if (flags & DIT_VEC_SILU_IN) z = silu(z);
    xs[k] = z;
  }
  __syncthreads();
  float xv[KC * 8];
#pragma unroll
  for (int j = 0; j < KC; ++j) {
    const float4* q = reinterpret_cast<const float4*>(xs + (lane + 32 * j) * 8);
    const float4 a = q[0], c = q[1];
    xv[j * 8 + 0] = a.x; xv[j * 8 + 1] = a.y; xv[j * 8 + 2] = a.z; xv[j * 8 + 3] = a.w;
    xv[j * 8 + 4] = c.x; xv[j * 8 + 5] = c.y; xv[j * 8 + 6] = c.z; xv[j * 8 + 7] = c.w;
  }
  int slot = 0;
  for (int64_t n = n0; n < N; n += nw) {
    {  // the slot consumed one row ago gets the row P - 1 ahead
      const int64_t nn = n + (int64_t)(P - 1) * nw;
      const int si = (slot == 0 ? P : slot) - 1;
      if (nn < N) {
        const uint4* src = row_ptr(nn);
#pragma unroll
        for (int j = 0; j < KC; ++j) cp_async16(&ring[si * row_chunks + lane + 32 * j], src + lane + 32 * j);
      }
      cp_async_commit();
    }
    const int jm = multi_find(p, n);
    const int64_t local = n - p.row_begin[jm];
    const float bv = p.bias[jm] ? __bfloat162float(p.bias[jm][local]) : 0.0f;
    cp_async_wait<P - 1>();
    float a0 = 0.f, a1 = 0.f;
#pragma unroll
    for (int j = 0; j < KC; ++j) {
      const uint4 u = ring[slot * row_chunks + lane + 32 * j];
      a0 = fmaf(bf16_lo(u.x), xv[j * 8 + 0], a0); a1 = fmaf(bf16_hi(u.x), xv[j * 8 + 1], a1);
      a0 = fmaf(bf16_lo(u.y), xv[j * 8 + 2], a0); a1 = fmaf(bf16_hi(u.y), xv[j * 8 + 3], a1);
      a0 = fmaf(bf16_lo(u.z), xv[j * 8 + 4], a0); a1 = fmaf(bf16_hi(u.z), xv[j * 8 + 5], a1);
      a0 = fmaf(bf16_lo(u.w), xv[j * 8 + 6], a0); a1 = fmaf(bf16_hi(u.w), xv[j * 8 + 7], a1);
    }
    const float a = warp_sum(a0 + a1) + bv;
    if (lane == 0) p.out[jm][local] = a;
    if (++slot == P) slot = 0;
  }
  cp_async_wait<0>();
}

// Every matrix of p in one pass with the loop above (one warp per row);
// out[j][n - row_begin[j]] = W_j[row] . f(x) + bias_j[row].
template <int KC>
__global__ void __launch_bounds__(512, 1) vec_rows_multi_kernel(const bf16* __restrict__ x,
                                                             const __grid_constant__ MultiLinear p, int flags) {
  vec_rows_loop<KC, 1>(
      x, 0, p.K, flags, (int64_t)p.row_begin[p.n_mats],
      [&](int64_t n) {
        const int j = multi_find(p, n);
        const int64_t local = n - p.row_begin[j];
        return VecRow{reinterpret_cast<const uint4*>(p.W[j] + local * p.K), p.bias[j], local, j};
      },
      [&](const VecRow& rw, int, float v) { p.out[rw.mat][rw.local] = v; });
}

// ---------------------------------------------------------------------------
// Bulk-copy staging of rows: 8 warps per CTA, each warp owns a 2-deep ring of
// row buffers in shared memory; lane 0 starts the copy of the warp's next row
// before the warp works on the current one.
// ---------------------------------------------------------------------------
constexpr int kRowWarps = 8;

// adaLN / vector x weight with bulk-copy staging of the weight rows (same
// warp-private 2-deep ring).  out[b][n] = sum_k W[n][k] f(x[b][k]) + bias[n].
template <int NB>
__global__ void __launch_bounds__(256) vec_linear_bulk_kernel(const bf16* __restrict__ x, int64_t ldx,
                                                              const bf16* __restrict__ W, int64_t ldw,
                                                              const bf16* __restrict__ bias, void* out, int64_t ldo,
                                                              int B, int N, int K, int flags, uint64_t wait_limit) {
  extern __shared__ __align__(128) uint8_t sm[];
  const int ROW_BYTES = K * 2;
  float* xs = reinterpret_cast<float*>(sm);  // [B][K]
  uint8_t* rings = sm + (size_t)B * K * 4;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* buf = rings + (size_t)warp * 2 * ROW_BYTES;
  uint64_t* bar = reinterpret_cast<uint64_t*>(rings + (size_t)kRowWarps * 2 * ROW_BYTES) + warp * 2;
  const int64_t nw = (int64_t)gridDim.x * kRowWarps;
  int64_t n = (int64_t)blockIdx.x * kRowWarps + warp;
  if (lane == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    fence_mbar_init();
    if (n < N) {
      mbar_arrive_expect_tx(&bar[0], ROW_BYTES);
      bulk_load(buf, W + n * ldw, ROW_BYTES, &bar[0]);
    }
  }
  for (int i = threadIdx.x; i < B * K; i += blockDim.x) {
    const int b = i / K, kk = i % K;
    float z = __bfloat162float(x[b * ldx + kk]);
    if (flags & DIT_VEC_SILU_IN) z = silu(z);
    xs[i] = z;
  }
  __syncthreads();
  int st = 0;
  uint32_t ph0 = 0, ph1 = 0;
  for (; n < N; n += nw) {
    const int64_t nn = n + nw;
    if (nn < N && lane == 0) {
      fence_proxy_async_smem();
      mbar_arrive_expect_tx(&bar[st ^ 1], ROW_BYTES);
      bulk_load(buf + (st ^ 1) * ROW_BYTES, W + nn * ldw, ROW_BYTES, &bar[st ^ 1]);
    }
    const uint32_t ph = st ? ph1 : ph0;
    bool ok = mbar_wait(&bar[st], ph, wait_limit, nullptr, SITE_ROWS);
    if (!__all_sync(0xffffffffu, ok)) {
      if (lane == 0 && nn < N) (void)mbar_wait(&bar[st ^ 1], st ? ph0 : ph1, wait_limit, nullptr, SITE_ROWS);
      break;
    }
    if (st) ph1 ^= 1; else ph0 ^= 1;
    const uint4* wp = reinterpret_cast<const uint4*>(buf + st * ROW_BYTES);
    float acc[NB];
#pragma unroll
    for (int b = 0; b < NB; ++b) acc[b] = 0.0f;
    for (int v = lane; v < K / 8; v += 32) {
      const uint4 u = wp[v];
      const float w8[8] = {bf16_lo(u.x), bf16_hi(u.x), bf16_lo(u.y), bf16_hi(u.y),
                           bf16_lo(u.z), bf16_hi(u.z), bf16_lo(u.w), bf16_hi(u.w)};
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        if (b < B) {
          const float4* xp = reinterpret_cast<const float4*>(xs + b * K + v * 8);
          const float4 x0 = xp[0], x1 = xp[1];
          acc[b] = fmaf(w8[0], x0.x, acc[b]); acc[b] = fmaf(w8[1], x0.y, acc[b]);
          acc[b] = fmaf(w8[2], x0.z, acc[b]); acc[b] = fmaf(w8[3], x0.w, acc[b]);
          acc[b] = fmaf(w8[4], x1.x, acc[b]); acc[b] = fmaf(w8[5], x1.y, acc[b]);
          acc[b] = fmaf(w8[6], x1.z, acc[b]); acc[b] = fmaf(w8[7], x1.w, acc[b]);
        }
      }
    }
    const float bv = bias ? __bfloat162float(bias[n]) : 0.0f;
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      if (b < B) {
        const float a = warp_sum(acc[b]) + bv;
        if (lane == 0) {
          if (flags & DIT_VEC_OUT_BF16)
            reinterpret_cast<bf16*>(out)[b * ldo + n] = __float2bfloat16_rn(a);
          else
            reinterpret_cast<float*>(out)[b * ldo + n] = a;
        }
      }
    }
    __syncwarp();
    st ^= 1;
  }
}

// ---------------------------------------------------------------------------
// Log-sum-exp merge of attention results over disjoint key sets (the ring
// attention hop merge of "compile_graph" (chenyy20.com) §5):
//   lse = log sum_j exp(lse_j),  o = sum_j exp(lse_j - lse) o_j.
// 16 threads per (batch, head, token) row of 128, 8 values each; weights in
// fp32.  Each thread reads its columns of every part before writing them, so
// the output may be one of the parts; the row's lse is written after the
// half-warp has read every part's lse, so lse_out may be one of them too.
// ---------------------------------------------------------------------------
constexpr int kMergeMaxParts = 8;
struct MergeParams {
  const bf16* o[kMergeMaxParts];
  const float* lse[kMergeMaxParts];
  int64_t ld[kMergeMaxParts];  // row stride of each part, elements
  bf16* out;
  float* lse_out;
  int64_t ld_out;
  int n, B, S, H;
};

template <int NP>  // bound on the number of parts (2, 4 or 8): every load is issued before any is used
__global__ void __launch_bounds__(256) attention_merge_kernel(const __grid_constant__ MergeParams p) {
  griddep_wait();
  griddep_launch_dependents();
  // grid (tokens / 16, H, B): 16 consecutive tokens of one (batch, head) per
  // CTA, so the lse accesses are contiguous and no index needs a division
  const int s = blockIdx.x * 16 + (threadIdx.x >> 4);
  const int sub = threadIdx.x & 15;
  const int h = blockIdx.y, b = blockIdx.z;
  const bool valid = s < p.S;
  const int64_t li = ((int64_t)b * p.H + h) * p.S + (valid ? s : 0);
  const int64_t bs = (int64_t)b * p.S + (valid ? s : 0);
  const int64_t col = (int64_t)h * 128 + sub * 8;
  float l[NP];
  uint4 u[NP];
#pragma unroll
  for (int j = 0; j < NP; ++j) {
    const bool on = valid && j < p.n;
    l[j] = on ? p.lse[j][li] : -INFINITY;
    u[j] = on ? *reinterpret_cast<const uint4*>(p.o[j] + bs * p.ld[j] + col) : make_uint4(0, 0, 0, 0);
  }
  float m = l[0];
#pragma unroll
  for (int j = 1; j < NP; ++j) m = fmaxf(m, l[j]);
  // every part of the row over an empty key set (lse = -inf): the union is
  // empty too, so o = 0 and lse = -inf instead of exp(-inf - -inf) = NaN
  const bool empty = m == -INFINITY;
  float den = 0.0f;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int j = 0; j < NP; ++j) {
    const float wj = (j < p.n && !empty) ? __expf(l[j] - m) : 0.0f;
    den += wj;
    acc[0] = fmaf(wj, bf16_lo(u[j].x), acc[0]); acc[1] = fmaf(wj, bf16_hi(u[j].x), acc[1]);
    acc[2] = fmaf(wj, bf16_lo(u[j].y), acc[2]); acc[3] = fmaf(wj, bf16_hi(u[j].y), acc[3]);
    acc[4] = fmaf(wj, bf16_lo(u[j].z), acc[4]); acc[5] = fmaf(wj, bf16_hi(u[j].z), acc[5]);
    acc[6] = fmaf(wj, bf16_lo(u[j].w), acc[6]); acc[7] = fmaf(wj, bf16_hi(u[j].w), acc[7]);
  }
  if (valid) {
    const float inv = empty ? 0.0f : 1.0f / den;
    *reinterpret_cast<uint4*>(p.out + bs * p.ld_out + col) =
        make_uint4(pack_bf16x2(acc[0] * inv, acc[1] * inv), pack_bf16x2(acc[2] * inv, acc[3] * inv),
                   pack_bf16x2(acc[4] * inv, acc[5] * inv), pack_bf16x2(acc[6] * inv, acc[7] * inv));
  }
  __syncwarp();
  if (valid && sub == 0 && p.lse_out != nullptr) p.lse_out[li] = empty ? -INFINITY : m + __logf(den);
}

// Self test of the FMA-pipe 2^x that the attention softmax uses on a part of
// its exponentials: y[i] = exp2_poly2 evaluated on the pair (x[2j], x[2j+1]).
__global__ void selftest_exp2_poly_kernel(const float* __restrict__ x, float* __restrict__ y, int64_t n) {
  const int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (2 * j >= n) return;
  const float x0 = x[2 * j], x1 = (2 * j + 1 < n) ? x[2 * j + 1] : 0.0f;
  const uint64_t r = exp2_poly2(x0, x1);
  y[2 * j] = f2_lo(r);
  if (2 * j + 1 < n) y[2 * j + 1] = f2_hi(r);
}

// ---------------------------------------------------------------------------
// QK RMSNorm + RoPE: one CTA of 128 threads per token row (grid = tokens x
// batch).  Thread t owns columns 8 (t & 15) .. +8 of every head vector, so its
// RoPE angles and norm scales are loaded once and reused for all 2H vectors
// (q heads, then k heads) that its group of 16 walks through, U at a time
// with every load issued first.  The 16 threads of a vector reduce its sum of
// squares with shuffles.  In place is safe: a vector is read in full before
// any of its columns is written.
// ---------------------------------------------------------------------------
template <int U>
__global__ void __launch_bounds__(128) qk_norm_rope_kernel(const bf16* q, const bf16* k, int64_t ld_in,
                                                           const bf16* __restrict__ q_scale,
                                                           const bf16* __restrict__ k_scale,
                                                           const float2* __restrict__ rope, bf16* q_out,
                                                           bf16* k_out, int64_t ld_out, int S, int H, float eps,
                                                           int do_norm) {
  const int sub = threadIdx.x & 15, grp = threadIdx.x >> 4;  // 8 groups of 16
  const int tok = blockIdx.x;
  const int64_t row = (int64_t)blockIdx.y * S + tok;
  float scq[8], sck[8];  // two named arrays: a runtime index would put them in local memory
#pragma unroll
  for (int wq = 0; wq < 2; ++wq) {
    const bf16* sp = wq ? k_scale : q_scale;
    float* sc = wq ? sck : scq;
    if (sp != nullptr) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(sp + sub * 8));
      sc[0] = bf16_lo(u.x); sc[1] = bf16_hi(u.x); sc[2] = bf16_lo(u.y); sc[3] = bf16_hi(u.y);
      sc[4] = bf16_lo(u.z); sc[5] = bf16_hi(u.z); sc[6] = bf16_lo(u.w); sc[7] = bf16_hi(u.w);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) sc[i] = 1.0f;
    }
  }
  float cs[4][2];
  if (rope != nullptr) {
    const float4* rp = reinterpret_cast<const float4*>(rope + (int64_t)tok * 64 + sub * 4);
    const float4 t0 = __ldg(rp), t1 = __ldg(rp + 1);
    cs[0][0] = t0.x; cs[0][1] = t0.y; cs[1][0] = t0.z; cs[1][1] = t0.w;
    cs[2][0] = t1.x; cs[2][1] = t1.y; cs[3][0] = t1.z; cs[3][1] = t1.w;
  }
  const int nv = 2 * H;
  for (int v0 = grp; v0 < nv; v0 += 8 * U) {
    uint4 u[U];
#pragma unroll
    for (int j = 0; j < U; ++j) {
      const int v = v0 + 8 * j;
      if (v < nv) {
        const int w = v >= H, h = v - w * H;
        u[j] = *reinterpret_cast<const uint4*>((w ? k : q) + row * ld_in + h * 128 + sub * 8);
      }
    }
#pragma unroll
    for (int j = 0; j < U; ++j) {
      const int v = v0 + 8 * j;
      const bool on = v < nv;  // uniform across the 16 threads of the vector
      const int w = v >= H, h = v - w * H;
      float x[8];
      if (on) {
        x[0] = bf16_lo(u[j].x); x[1] = bf16_hi(u[j].x); x[2] = bf16_lo(u[j].y); x[3] = bf16_hi(u[j].y);
        x[4] = bf16_lo(u[j].z); x[5] = bf16_hi(u[j].z); x[6] = bf16_lo(u[j].w); x[7] = bf16_hi(u[j].w);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) x[i] = 0.0f;
      }
      float ss = 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) ss = fmaf(x[i], x[i], ss);
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      if (!on) continue;
      const float r = do_norm ? rsqrtf(ss * (1.0f / 128.0f) + eps) : 1.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) x[i] = x[i] * r * (w ? sck[i] : scq[i]);
      if (rope != nullptr) {
#pragma unroll
        for (int pp = 0; pp < 4; ++pp) {
          const float a = x[2 * pp], bb = x[2 * pp + 1], c = cs[pp][0], sn = cs[pp][1];
          x[2 * pp] = a * c - bb * sn;
          x[2 * pp + 1] = a * sn + bb * c;
        }
      }
      uint4 o4;
      o4.x = pack_bf16x2(x[0], x[1]); o4.y = pack_bf16x2(x[2], x[3]);
      o4.z = pack_bf16x2(x[4], x[5]); o4.w = pack_bf16x2(x[6], x[7]);
      *reinterpret_cast<uint4*>((w ? k_out : q_out) + row * ld_out + h * 128 + sub * 8) = o4;
    }
  }
}

// ---------------------------------------------------------------------------
// RoPE table: rope[t][p] = (cos, sin) of ids[t][a] * theta^(-2j / (2 P_a)).
// ---------------------------------------------------------------------------
__global__ void rope_table_kernel(const int32_t* __restrict__ ids, int S, int n_axes, int p0, int p1, int p2,
                                  double theta, float2* __restrict__ out) {
  const int n_pairs = p0 + p1 + p2;
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (int64_t)S * n_pairs) return;
  const int t = (int)(i / n_pairs);
  const int p = (int)(i % n_pairs);
  int a, j, pa;
  if (p < p0) { a = 0; j = p; pa = p0; }
  else if (p < p0 + p1) { a = 1; j = p - p0; pa = p1; }
  else { a = 2; j = p - p0 - p1; pa = p2; }
  double pos = (a < n_axes) ? (double)ids[(int64_t)t * n_axes + a] : 0.0;
  double omega = pow(theta, -2.0 * (double)j / (double)(2 * pa));
  double s, c;
  sincos(pos * omega, &s, &c);
  out[i] = make_float2((float)c, (float)s);
}

// ---------------------------------------------------------------------------
// Vector x weight (adaLN modulation, timestep MLP): one warp per output
// feature, 16-byte streaming loads of the weight row, the (mapped) input
// vector staged in shared memory as fp32.
// ---------------------------------------------------------------------------
template <int NB>
__global__ void __launch_bounds__(256) vec_linear_kernel(const bf16* __restrict__ x, int64_t ldx,
                                                         const bf16* __restrict__ W, int64_t ldw,
                                                         const bf16* __restrict__ bias, void* out,
                                                         int64_t ldo, int B, int N, int K, int flags) {
  extern __shared__ float xs[];  // [B][K]
  for (int i = threadIdx.x; i < B * K; i += blockDim.x) {
    const int b = i / K, kk = i % K;
    float z = __bfloat162float(x[b * ldx + kk]);
    if (flags & DIT_VEC_SILU_IN) z = silu(z);
    xs[i] = z;
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  for (int n = blockIdx.x * nwarps + warp; n < N; n += gridDim.x * nwarps) {
    float acc[NB];
#pragma unroll
    for (int b = 0; b < NB; ++b) acc[b] = 0.0f;
    const bf16* wr = W + (int64_t)n * ldw;
    if (K <= 16 * 256) {
      // issue the whole row's loads first (up to 16 x 16 bytes per lane)
      uint4 wv[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int k0 = j * 256 + lane * 8;
        wv[j] = (k0 < K) ? __ldcs(reinterpret_cast<const uint4*>(wr + k0)) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int k0 = j * 256 + lane * 8;
        if (k0 < K) {
          const uint4 u = wv[j];
          const float w[8] = {bf16_lo(u.x), bf16_hi(u.x), bf16_lo(u.y), bf16_hi(u.y),
                              bf16_lo(u.z), bf16_hi(u.z), bf16_lo(u.w), bf16_hi(u.w)};
#pragma unroll
          for (int b = 0; b < NB; ++b) {
            if (b < B) {
              const float4* xp = reinterpret_cast<const float4*>(xs + b * K + k0);
              const float4 x0 = xp[0], x1 = xp[1];
              acc[b] = fmaf(w[0], x0.x, acc[b]); acc[b] = fmaf(w[1], x0.y, acc[b]);
              acc[b] = fmaf(w[2], x0.z, acc[b]); acc[b] = fmaf(w[3], x0.w, acc[b]);
              acc[b] = fmaf(w[4], x1.x, acc[b]); acc[b] = fmaf(w[5], x1.y, acc[b]);
              acc[b] = fmaf(w[6], x1.z, acc[b]); acc[b] = fmaf(w[7], x1.w, acc[b]);
            }
          }
        }
      }
    } else
    for (int k0 = lane * 8; k0 < K; k0 += 256) {
      uint4 u = __ldcs(reinterpret_cast<const uint4*>(wr + k0));
      float w[8] = {bf16_lo(u.x), bf16_hi(u.x), bf16_lo(u.y), bf16_hi(u.y),
                    bf16_lo(u.z), bf16_hi(u.z), bf16_lo(u.w), bf16_hi(u.w)};
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        if (b < B) {
          const float4* xp = reinterpret_cast<const float4*>(xs + b * K + k0);
          float4 x0 = xp[0], x1 = xp[1];
          acc[b] = fmaf(w[0], x0.x, acc[b]); acc[b] = fmaf(w[1], x0.y, acc[b]);
          acc[b] = fmaf(w[2], x0.z, acc[b]); acc[b] = fmaf(w[3], x0.w, acc[b]);
          acc[b] = fmaf(w[4], x1.x, acc[b]); acc[b] = fmaf(w[5], x1.y, acc[b]);
          acc[b] = fmaf(w[6], x1.z, acc[b]); acc[b] = fmaf(w[7], x1.w, acc[b]);
        }
      }
    }
    const float bv = bias ? __bfloat162float(bias[n]) : 0.0f;
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      if (b < B) {
        float a = warp_sum(acc[b]) + bv;
        if (lane == 0) {
          if (flags & DIT_VEC_OUT_BF16)
            reinterpret_cast<bf16*>(out)[b * ldo + n] = __float2bfloat16_rn(a);
          else
            reinterpret_cast<float*>(out)[b * ldo + n] = a;
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Loop helpers (Flux top level): timestep embedding, patchify, Euler step.
// ---------------------------------------------------------------------------

// emb = [cos(1000 t f_k), sin(1000 t f_k)], f_k = 10000^(-k/half); bf16 out.
// t is read from tsched[step] (device, fp32 schedule) so one graph node per
// step needs no host value.
__global__ void timestep_embed_kernel(const float* __restrict__ tsched, int step, int dim, bf16* __restrict__ emb) {
  const int half = dim / 2;
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= half) return;
  const double t = (double)tsched[step];
  const double f = pow(10000.0, -(double)k / (double)half);
  double s, c;
  sincos(1000.0 * t * f, &s, &c);
  emb[k] = __float2bfloat16_rn((float)c);
  emb[half + k] = __float2bfloat16_rn((float)s);
}

// latent [C][2Hg][2Wg] bf16 -> state tokens [Hg*Wg][4C] fp32 and bf16 copy.
__global__ void patchify_kernel(const bf16* __restrict__ lat, int C, int Hg, int Wg, float* __restrict__ state,
                                bf16* __restrict__ tok) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int F = 4 * C;
  if (i >= (int64_t)Hg * Wg * F) return;
  const int t = (int)(i / F), f = (int)(i % F);
  const int h = t / Wg, w = t % Wg;
  const int c = f / 4, ph = (f / 2) % 2, pw = f % 2;
  const bf16 v = lat[((int64_t)c * 2 * Hg + 2 * h + ph) * (2 * Wg) + 2 * w + pw];
  state[i] = __bfloat162float(v);
  tok[i] = v;
}

// state tokens [Hg*Wg][4C] fp32 -> latent [C][2Hg][2Wg] fp32.
__global__ void unpatchify_kernel(const float* __restrict__ state, int C, int Hg, int Wg,
                                  float* __restrict__ lat) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int F = 4 * C;
  if (i >= (int64_t)Hg * Wg * F) return;
  const int t = (int)(i / F), f = (int)(i % F);
  const int h = t / Wg, w = t % Wg;
  const int c = f / 4, ph = (f / 2) % 2, pw = f % 2;
  lat[((int64_t)c * 2 * Hg + 2 * h + ph) * (2 * Wg) + 2 * w + pw] = state[i];
}

// x += (t_{i+1} - t_i) v, state fp32; also refresh the bf16 copy fed to img_in.
// vhist (optional): keep the model velocity of this step for the step cache.
// vu != null: classifier-free guidance, v = vu + g (v - vu) in fp32.
__global__ void euler_kernel(float* __restrict__ state, bf16* __restrict__ tok, const bf16* __restrict__ v,
                             int64_t n, const float* __restrict__ tsched, int step, float* __restrict__ vhist,
                             const bf16* __restrict__ vu = nullptr, float g = 1.0f) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const float dt = tsched[step + 1] - tsched[step];
  float vi = __bfloat162float(v[i]);
  if (vu != nullptr) {
    const float u = __bfloat162float(vu[i]);
    vi = fmaf(g, vi - u, u);
  }
  if (vhist != nullptr) vhist[i] = vi;
  const float s = fmaf(dt, vi, state[i]);
  state[i] = s;
  tok[i] = __float2bfloat16_rn(s);
}

// Cached step: v = ca * va + cb * vb from kept model velocities (vb may be
// null), then the same Euler update.
__global__ void euler_cached_kernel(float* __restrict__ state, bf16* __restrict__ tok, const float* __restrict__ va,
                                    const float* __restrict__ vb, float ca, float cb, int64_t n,
                                    const float* __restrict__ tsched, int step) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const float dt = tsched[step + 1] - tsched[step];
  float v = ca * va[i];
  if (vb != nullptr) v = fmaf(cb, vb[i], v);
  const float s = fmaf(dt, v, state[i]);
  state[i] = s;
  tok[i] = __float2bfloat16_rn(s);
}

// Wait on a barrier nothing arrives on; must time out and record the error.
__global__ void selftest_wait_kernel(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    (void)mbar_wait(&bar, 0, limit_ns, &abort_flag, SITE_SELFTEST);
  }
  __syncthreads();
}

}  // namespace dit

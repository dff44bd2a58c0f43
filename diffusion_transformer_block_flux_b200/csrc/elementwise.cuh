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

__device__ __forceinline__ float block_sum(float v, float* red) {
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31, nw = blockDim.x >> 5;
  v = warp_sum(v);
  __syncthreads();  // red may still be read from a previous call
  if (l == 0) red[w] = v;
  __syncthreads();
  float t = (l < nw) ? red[l] : 0.0f;
  return warp_sum(t);
}

// ---------------------------------------------------------------------------
// LayerNorm + modulate: one CTA per row, 8 bf16 (16 bytes) per thread.
// Two-pass statistics from registers (mean, then centred second moment).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024) modulate_norm_kernel(const bf16* __restrict__ x, int64_t ldx,
                                                             const float* __restrict__ shift,
                                                             const float* __restrict__ scale,
                                                             int64_t mod_stride, bf16* __restrict__ y,
                                                             int64_t ldy, int S, int D, float eps) {
  __shared__ float red[32];
  const int64_t row = blockIdx.x;
  const int b = (int)(row / S);
  const int c0 = threadIdx.x * 8;
  const bool active = c0 < D;
  float v[8];
  if (active) {
    uint4 u = __ldcs(reinterpret_cast<const uint4*>(x + row * ldx + c0));
    v[0] = bf16_lo(u.x); v[1] = bf16_hi(u.x); v[2] = bf16_lo(u.y); v[3] = bf16_hi(u.y);
    v[4] = bf16_lo(u.z); v[5] = bf16_hi(u.z); v[6] = bf16_lo(u.w); v[7] = bf16_hi(u.w);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = 0.0f;
  }
  float s = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) s += v[i];
  const float mean = block_sum(s, red) / (float)D;
  float q = 0.0f;
  if (active) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float d = v[i] - mean;
      q = fmaf(d, d, q);
    }
  }
  const float var = block_sum(q, red) / (float)D;
  const float rstd = rsqrtf(var + eps);
  if (!active) return;
  float sh[8], sc[8];
  if (shift != nullptr) {
    const float4* ps = reinterpret_cast<const float4*>(shift + b * mod_stride + c0);
    const float4* pc = reinterpret_cast<const float4*>(scale + b * mod_stride + c0);
    float4 a0 = __ldg(ps), a1 = __ldg(ps + 1), b0 = __ldg(pc), b1 = __ldg(pc + 1);
    sh[0] = a0.x; sh[1] = a0.y; sh[2] = a0.z; sh[3] = a0.w; sh[4] = a1.x; sh[5] = a1.y; sh[6] = a1.z; sh[7] = a1.w;
    sc[0] = b0.x; sc[1] = b0.y; sc[2] = b0.z; sc[3] = b0.w; sc[4] = b1.x; sc[5] = b1.y; sc[6] = b1.z; sc[7] = b1.w;
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) { sh[i] = 0.0f; sc[i] = 0.0f; }
  }
  float o[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) o[i] = fmaf(1.0f + sc[i], (v[i] - mean) * rstd, sh[i]);
  uint4 w;
  w.x = pack_bf16x2(o[0], o[1]); w.y = pack_bf16x2(o[2], o[3]);
  w.z = pack_bf16x2(o[4], o[5]); w.w = pack_bf16x2(o[6], o[7]);
  *reinterpret_cast<uint4*>(y + row * ldy + c0) = w;
}

// ---------------------------------------------------------------------------
// QK RMSNorm + RoPE: 16 threads per (token, head, q|k) vector of 128, each
// thread 8 elements = 4 rotation pairs.  In place is safe: a group reads its
// whole vector before any thread writes.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) qk_norm_rope_kernel(const bf16* q, const bf16* k, int64_t ld_in,
                                                           const bf16* __restrict__ q_scale,
                                                           const bf16* __restrict__ k_scale,
                                                           const float2* __restrict__ rope, bf16* q_out,
                                                           bf16* k_out, int64_t ld_out, int S, int H,
                                                           int64_t n_vecs, float eps, int do_norm) {
  const int64_t gid = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 4;
  const int sub = threadIdx.x & 15;
  const bool valid = gid < n_vecs;
  const int which = (int)(gid & 1);  // 0: q, 1: k
  const int64_t hv = gid >> 1;
  const int h = (int)(hv % H);
  const int64_t row = hv / H;
  const int tok = (int)(row % S);
  const bf16* src = (which ? k : q) + row * ld_in + h * 128 + sub * 8;
  bf16* dst = (which ? k_out : q_out) + row * ld_out + h * 128 + sub * 8;
  float v[8];
  if (valid) {
    uint4 u = *reinterpret_cast<const uint4*>(src);
    v[0] = bf16_lo(u.x); v[1] = bf16_hi(u.x); v[2] = bf16_lo(u.y); v[3] = bf16_hi(u.y);
    v[4] = bf16_lo(u.z); v[5] = bf16_hi(u.z); v[6] = bf16_lo(u.w); v[7] = bf16_hi(u.w);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = 0.0f;
  }
  float ss = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) ss = fmaf(v[i], v[i], ss);
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if (!valid) return;
  const float r = do_norm ? rsqrtf(ss * (1.0f / 128.0f) + eps) : 1.0f;
  const bf16* sp = which ? k_scale : q_scale;
  float sc[8];
  if (sp != nullptr) {
    uint4 u = __ldg(reinterpret_cast<const uint4*>(sp + sub * 8));
    sc[0] = bf16_lo(u.x); sc[1] = bf16_hi(u.x); sc[2] = bf16_lo(u.y); sc[3] = bf16_hi(u.y);
    sc[4] = bf16_lo(u.z); sc[5] = bf16_hi(u.z); sc[6] = bf16_lo(u.w); sc[7] = bf16_hi(u.w);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) sc[i] = 1.0f;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = v[i] * r * sc[i];
  if (rope != nullptr) {
    const float4* rp = reinterpret_cast<const float4*>(rope + (int64_t)tok * 64 + sub * 4);
    float4 t0 = __ldg(rp), t1 = __ldg(rp + 1);
    float cs[4][2] = {{t0.x, t0.y}, {t0.z, t0.w}, {t1.x, t1.y}, {t1.z, t1.w}};
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const float a = v[2 * p], bb = v[2 * p + 1], c = cs[p][0], s = cs[p][1];
      v[2 * p] = a * c - bb * s;
      v[2 * p + 1] = a * s + bb * c;
    }
  }
  uint4 w;
  w.x = pack_bf16x2(v[0], v[1]); w.y = pack_bf16x2(v[2], v[3]);
  w.z = pack_bf16x2(v[4], v[5]); w.w = pack_bf16x2(v[6], v[7]);
  *reinterpret_cast<uint4*>(dst) = w;
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
__global__ void euler_kernel(float* __restrict__ state, bf16* __restrict__ tok, const bf16* __restrict__ v,
                             int64_t n, const float* __restrict__ tsched, int step) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const float dt = tsched[step + 1] - tsched[step];
  const float s = fmaf(dt, __bfloat162float(v[i]), state[i]);
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

// Flash attention, head_dim 128, on tcgen05 tensor cores with TMEM
// accumulators and an online softmax.
//
// Page: "compile_graph" (chenyy20.com), §2 — joint full attention over the
// 4608-token text|image sequence, 24 heads x 128, bf16, run by a flash
// backend; §6.3 — operands laid out (B, S, H, D).  No mask.
//
// One CTA = one (batch, head) and two 128-row query tiles Q0, Q1 that
// ping-pong: while one softmax warpgroup turns its score tile into
// probabilities, the tensor core computes the other tile's scores and PV.
//   warps 0-3  softmax + epilogue for Q0 (thread = query row = TMEM lane)
//   warps 4-7  softmax + epilogue for Q1
//   warp 8     TMA producer: Q0, Q1 once; K_j, V_j through 2-stage rings
//   warp 9     TMEM allocator + single-thread MMA issuer
// TMEM (512 columns): S0 [0,128) S1 [128,256) O0 [256,384) O1 [384,512).
// P_k (bf16 pairs) overwrites the first 64 columns of S_k after the softmax
// has read S_k into registers; the next S_k MMA is issued after the PV MMA
// that reads P_k, and tcgen05 MMAs of one CTA execute in issue order.
// A commit after S_k(j+1) therefore also covers PV_k(j): once a softmax
// warpgroup sees S_k(j+1), O_k is stable and may be rescaled in place.
#pragma once

#include "common.cuh"

namespace dit {
namespace attn {

constexpr int BQ = 128;
constexpr int BKV = 128;
constexpr int HD = 128;
constexpr int TILE_BYTES = 128 * HD * 2;  // 32 KB: two 64-column swizzled halves
constexpr int HALF_BYTES = TILE_BYTES / 2;
constexpr int NUM_THREADS = 320;
constexpr int OFF_Q = 0;                        // Q0, Q1
constexpr int OFF_K = 2 * TILE_BYTES;           // K[2]
constexpr int OFF_V = 4 * TILE_BYTES;           // V[2]
constexpr int OFF_BAR = 6 * TILE_BYTES;
constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t IDESC_QK = idesc_bf16(128, 128, 0, 0);  // Q, K both K-major (d contiguous)
constexpr uint32_t IDESC_PV = idesc_bf16(128, 128, 0, 1);  // P from TMEM, V MN-major (d contiguous)

struct Params {
  bf16* o;
  int64_t ldo;
  float* lse;
  int Sq, Skv, H;
  float scale_log2;  // softmax_scale * log2(e)
};

__global__ void __launch_bounds__(NUM_THREADS, 1)
    attention_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, Params p, uint64_t wait_limit) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;   // [2]
  uint64_t* k_empty = bars + 3;  // [2]
  uint64_t* v_full = bars + 5;   // [2]
  uint64_t* v_empty = bars + 7;  // [2]
  uint64_t* s_full = bars + 9;   // [2]
  uint64_t* p_full = bars + 11;  // [2]
  uint64_t* o_full = bars + 13;  // [2]
  uint64_t* drain = bars + 15;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 16);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int head = blockIdx.y;
  const int batch = blockIdx.z;
  const int q_row0 = blockIdx.x * 2 * BQ;
  const int n_kv = (p.Skv + BKV - 1) / BKV;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], 4);  // one arrival per softmax warp of the tile
      mbar_init(&o_full[s], 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 8) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      const int x0 = head * HD;
      mbar_arrive_expect_tx(q_full, 2 * TILE_BYTES);
      for (int t = 0; t < 2; ++t)
        for (int hf = 0; hf < 2; ++hf)
          tma_load_3d(smem + OFF_Q + t * TILE_BYTES + hf * HALF_BYTES, &tmQ, q_full, x0 + hf * 64,
                      q_row0 + t * BQ, batch);
      uint32_t k_issued = 0, v_issued = 0, k_par = 0, v_par = 0;
      bool ok = true;
      for (int j = 0; j < n_kv && ok; ++j) {
        const int st = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        if (!mbar_wait(&k_empty[st], ph ^ 1, wait_limit, abort_flag, SITE_ATTN_LOAD)) { ok = false; break; }
        mbar_arrive_expect_tx(&k_full[st], TILE_BYTES);
        for (int hf = 0; hf < 2; ++hf)
          tma_load_3d(smem + OFF_K + st * TILE_BYTES + hf * HALF_BYTES, &tmK, &k_full[st], x0 + hf * 64,
                      j * BKV, batch);
        k_issued |= 1u << st;
        k_par = (k_par & ~(1u << st)) | (ph << st);
        if (!mbar_wait(&v_empty[st], ph ^ 1, wait_limit, abort_flag, SITE_ATTN_LOAD)) { ok = false; break; }
        mbar_arrive_expect_tx(&v_full[st], TILE_BYTES);
        for (int hf = 0; hf < 2; ++hf)
          tma_load_3d(smem + OFF_V + st * TILE_BYTES + hf * HALF_BYTES, &tmV, &v_full[st], x0 + hf * 64,
                      j * BKV, batch);
        v_issued |= 1u << st;
        v_par = (v_par & ~(1u << st)) | (ph << st);
      }
      // Q always landed or is landing: wait for it too before leaving.
      (void)mbar_wait(q_full, 0, wait_limit, nullptr, SITE_ATTN_DRAIN);
      if (!ok) {
        for (int s = 0; s < 2; ++s) {
          if (k_issued & (1u << s)) (void)mbar_wait(&k_full[s], (k_par >> s) & 1u, wait_limit, nullptr, SITE_ATTN_DRAIN);
          if (v_issued & (1u << s)) (void)mbar_wait(&v_full[s], (v_par >> s) & 1u, wait_limit, nullptr, SITE_ATTN_DRAIN);
        }
      }
    }
  } else if (warp == 9) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      const uint32_t sQ0 = smem_u32(smem + OFF_Q);
      bool ok = true;
      bool issued = false;
      auto issue_qk = [&](int t, int kst) {
        const uint32_t kb = smem_u32(smem + OFF_K + kst * TILE_BYTES);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (uint32_t)((kk >> 2) * HALF_BYTES + (kk & 3) * 32);
          umma_ss(tmem_base + (uint32_t)(t * 128), sdesc_sw128(sQ0 + (uint32_t)(t * TILE_BYTES) + off, 16, 1024),
                  sdesc_sw128(kb + off, 16, 1024), IDESC_QK, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int t, int vst, bool acc) {
        const uint32_t vb = smem_u32(smem + OFF_V + vst * TILE_BYTES);
#pragma unroll
        for (int kk = 0; kk < BKV / 16; ++kk) {
          // A: P_t in TMEM, 16 keys = 8 columns of bf16 pairs.
          // B: V MN-major; 64-d halves HALF_BYTES apart (LBO), 8-key groups 1024 B apart (SBO).
          umma_ts(tmem_base + 256u + (uint32_t)(t * 128), tmem_base + (uint32_t)(t * 128 + kk * 8),
                  sdesc_sw128(vb + (uint32_t)(kk * 2048), HALF_BYTES, 1024), IDESC_PV, (acc || kk > 0) ? 1u : 0u);
        }
      };
      if (!mbar_wait(q_full, 0, wait_limit, abort_flag, SITE_ATTN_MMA)) ok = false;
      if (ok && !mbar_wait(&k_full[0], 0, wait_limit, abort_flag, SITE_ATTN_MMA)) ok = false;
      if (ok) {
        tc_fence_after();
        issue_qk(0, 0);
        umma_commit(&s_full[0]);
        issue_qk(1, 0);
        umma_commit(&s_full[1]);
        umma_commit(&k_empty[0]);
        issued = true;
      }
      for (int j = 0; j < n_kv && ok; ++j) {
        const int st = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        const bool has_next = j + 1 < n_kv;
        const int nst = (j + 1) & 1;
        const uint32_t nph = ((j + 1) >> 1) & 1;
        if (!mbar_wait(&v_full[st], ph, wait_limit, abort_flag, SITE_ATTN_MMA)) { ok = false; break; }
        if (!mbar_wait(&p_full[0], j & 1, wait_limit, abort_flag, SITE_ATTN_MMA)) { ok = false; break; }
        tc_fence_after();
        issue_pv(0, st, j > 0);
        if (has_next) {
          if (!mbar_wait(&k_full[nst], nph, wait_limit, abort_flag, SITE_ATTN_MMA)) { ok = false; break; }
          tc_fence_after();
          issue_qk(0, nst);
          umma_commit(&s_full[0]);
        }
        if (!mbar_wait(&p_full[1], j & 1, wait_limit, abort_flag, SITE_ATTN_MMA)) { ok = false; break; }
        tc_fence_after();
        issue_pv(1, st, j > 0);
        umma_commit(&v_empty[st]);
        if (has_next) {
          issue_qk(1, nst);
          umma_commit(&s_full[1]);
          umma_commit(&k_empty[nst]);
        }
      }
      if (ok) {
        umma_commit(&o_full[0]);
        umma_commit(&o_full[1]);
      } else if (issued) {
        umma_commit(drain);
        (void)mbar_wait(drain, 0, wait_limit, nullptr, SITE_ATTN_DRAIN);
      }
    }
  } else {
    // ---------------- softmax warpgroups ----------------
    const int t = warp >> 2;          // which query tile
    const int quad = warp & 3;        // TMEM lane quadrant
    const int row = quad * 32 + lane; // query row within the tile
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t tS = tmem_base + lane_off + (uint32_t)(t * 128);
    const uint32_t tO = tmem_base + lane_off + 256u + (uint32_t)(t * 128);
    const float sl2 = p.scale_log2;
    // Running max of the scaled logits (log2 units).  It is raised lazily:
    // only when a tile's max exceeds it by more than 8, so P stays <= 2^8 and
    // O is rescaled rarely (each thread owns its row, so the decision is
    // per row; the TMEM round trip runs when any row of the warp needs it).
    float m_run = -INFINITY;
    float l_run = 0.0f;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      ok = mbar_wait(&s_full[t], j & 1, wait_limit, abort_flag, SITE_ATTN_SOFTMAX);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      uint32_t r[4][32];
      tmem_ld32_nowait(tS + 0u, r[0]);
      tmem_ld32_nowait(tS + 32u, r[1]);
      tmem_ld32_nowait(tS + 64u, r[2]);
      tmem_ld32_nowait(tS + 96u, r[3]);
      tmem_wait_ld();
      reg_fence32(r[0]);
      reg_fence32(r[1]);
      reg_fence32(r[2]);
      reg_fence32(r[3]);
      const int valid = p.Skv - j * BKV;  // keys of this tile that exist
      if (valid < BKV) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (c * 32 + i >= valid) r[c][i] = __float_as_uint(-INFINITY);
      }
      // row max: four independent chains of 3-input max
      float mx[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float a = fmaxf(__uint_as_float(r[c][0]), __uint_as_float(r[c][1]));
#pragma unroll
        for (int i = 2; i < 32; i += 2) a = max3f(a, __uint_as_float(r[c][i]), __uint_as_float(r[c][i + 1]));
        mx[c] = a;
      }
      const float m_tile = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * sl2;
      const bool need = m_tile > m_run + 8.0f;  // always true on the first tile
      const float m_new = need ? m_tile : m_run;
      const float alpha = need ? ex2_fast(m_run - m_new) : 1.0f;  // 0 on the first tile
      const uint64_t sl2x2 = f2_pack(sl2, sl2);
      const uint64_t negx2 = f2_pack(-m_new, -m_new);
      uint64_t sum2[2] = {0ull, 0ull};  // packed (even, odd) partial sums, two chains
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          // x = s * scale * log2(e) - m for the pair (2i, 2i+1): one packed FMA
          const uint64_t x = f2_fma((uint64_t)r[c][2 * i] | ((uint64_t)r[c][2 * i + 1] << 32), sl2x2, negx2);
          uint64_t pp;
          if ((i & 3) == 3) {  // a quarter of the exponentials on the FMA pipe
            pp = exp2_poly2(f2_lo(x), f2_hi(x));
          } else {
            pp = f2_pack(ex2_fast(f2_lo(x)), ex2_fast(f2_hi(x)));
          }
          sum2[i & 1] = f2_add(sum2[i & 1], pp);
          pk[i] = pack_bf16x2(f2_lo(pp), f2_hi(pp));
        }
        tmem_st16(tS + (uint32_t)(c * 16), pk);
      }
      const uint64_t st2 = f2_add(sum2[0], sum2[1]);
      l_run = l_run * alpha + (f2_lo(st2) + f2_hi(st2));
      // Rescale O_t when any row of this warp raised its max (O_t is stable:
      // the commit we waited on covers the previous PV into O_t).
      if (j > 0 && __any_sync(0xffffffffu, need)) {
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + (uint32_t)(c * 32), o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(tO + (uint32_t)(c * 32), o);
        }
      }
      m_run = m_new;
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();  // every lane's P (and O) stores are complete before the warp's one arrival
      if (lane == 0) mbar_arrive(&p_full[t]);
    }
    if (ok) {
      ok = mbar_wait(&o_full[t], 0, wait_limit, abort_flag, SITE_ATTN_SOFTMAX);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      tc_fence_after();
      const int qi = q_row0 + t * BQ + row;
      const float inv_l = 1.0f / l_run;
      bf16* orow = p.o + ((int64_t)batch * p.Sq + qi) * p.ldo + head * HD;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(tO + (uint32_t)(c * 32), r);
        if (qi < p.Sq) {
          uint4* dp = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(r[8 * q + 0]) * inv_l, __uint_as_float(r[8 * q + 1]) * inv_l);
            w.y = pack_bf16x2(__uint_as_float(r[8 * q + 2]) * inv_l, __uint_as_float(r[8 * q + 3]) * inv_l);
            w.z = pack_bf16x2(__uint_as_float(r[8 * q + 4]) * inv_l, __uint_as_float(r[8 * q + 5]) * inv_l);
            w.w = pack_bf16x2(__uint_as_float(r[8 * q + 6]) * inv_l, __uint_as_float(r[8 * q + 7]) * inv_l);
            dp[q] = w;
          }
        }
      }
      if (p.lse != nullptr && qi < p.Sq)
        p.lse[((int64_t)batch * p.H + head) * p.Sq + qi] = (m_run + __log2f(l_run)) * 0.6931471805599453f;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 9) tmem_dealloc(tmem_base, TMEM_COLS);
}

}  // namespace attn
}  // namespace dit

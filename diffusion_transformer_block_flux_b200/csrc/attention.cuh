// Flash attention, head_dim 128, on tcgen05 tensor cores with TMEM
// accumulators and an online softmax.
//
// Page: "compile_graph" (chenyy20.com), §2 — joint full attention over the
// 4608-token text|image sequence, 24 heads x 128, bf16, run by a flash
// backend; §6.3 — operands laid out (B, S, H, D).  No mask.
//
// One CTA = one (batch, head, key range) and two 128-row query tiles Q0, Q1.
//   warps 0-3  softmax + epilogue for Q0 (thread = query row = TMEM lane)
//   warps 4-7  softmax + epilogue for Q1
//   warp 8     TMA producer: Q0, Q1 once; K_j, V_j through 2-stage rings
//   warp 9     TMEM allocator + MMA issuer (the whole warp runs the loop,
//              one elected lane issues each tcgen05 instruction)
// TMEM (512 columns): S [0,128) shared by both tiles, P0 [128,192),
// P1 [192,256) (bf16 pairs), O0 [256,384), O1 [384,512).
// The score tile S is the only buffer the two tiles share, and a tile's
// softmax holds it only until its scores are in registers: it then frees S
// (s_free) and the MMA issuer computes the other tile's next scores into it
// while the exponentials run.  P_t has its own columns, so the PV product of
// step j and the scores of step j + 1 never wait for each other; a tile
// only waits for its previous PV (p_free) before writing P_t again or
// rescaling O_t.  Each tile's softmax warps therefore run back to back, and
// the tensor core works through QK0 QK1 PV0 PV1 per key tile in the order
//   QK0(j+1), PV0(j), QK1(j+1), PV1(j).
#pragma once

#include "common.cuh"

namespace dit {

// Most key splits one split launch takes (dit_attention_split); with the
// running result they make at most five parts for the merge.
constexpr int kAttnMaxSplits = 4;

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
constexpr uint32_t COL_S = 0, COL_P = 128, COL_O = 256;  // P_t at COL_P + 64 t, O_t at COL_O + 128 t
constexpr uint32_t IDESC_QK = idesc_bf16(128, 128, 0, 0);  // Q, K both K-major (d contiguous)
constexpr uint32_t IDESC_PV = idesc_bf16(128, 128, 0, 1);  // P from TMEM, V MN-major (d contiguous)

struct Params {
  bf16* o;
  int64_t ldo;
  float* lse;
  int Sq, Skv, H;
  float scale_log2;  // softmax_scale * log2(e)
  // 1: o and lse hold a running result over other keys on entry; this
  // launch's result is merged into it by log-sum-exp (a ring hop)
  int accumulate;
  // Key split: blockIdx.z = batch * splits + s, and split s attends to keys
  // [s kv_per_split, min(Skv, (s + 1) kv_per_split)) (never empty), writing
  // its partial result to o + s o_split_stride and lse + s lse_split_stride.
  // splits = 1, kv_per_split = Skv: the plain launch.
  int splits;
  int kv_per_split;  // a multiple of BKV when splits > 1
  int64_t o_split_stride;
  int64_t lse_split_stride;
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
  uint64_t* s_full = bars + 9;   // [2] scores of tile t are in S
  uint64_t* s_free = bars + 11;  // the tile that last received S has loaded it
  uint64_t* p_full = bars + 12;  // [2] P_t written
  uint64_t* p_free = bars + 14;  // [2] the PV that read P_t is done (O_t stable)
  uint64_t* o_full = bars + 16;  // [2]
  uint64_t* drain = bars + 18;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 19);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int head = blockIdx.y;
  const int split = (int)blockIdx.z % p.splits;
  const int batch = (int)blockIdx.z / p.splits;
  const int kv0 = split * p.kv_per_split;                    // first key of this CTA's range
  const int kv_len = min(p.Skv - kv0, p.kv_per_split);       // keys in the range (>= 1)
  const int q_row0 = blockIdx.x * 2 * BQ;
  const int n_kv = (kv_len + BKV - 1) / BKV;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 4);  // the four warps of tile 1, once they hold the scores of the last QK
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], 4);  // one arrival per softmax warp of the tile
      mbar_init(&p_free[s], 1);
      mbar_init(&o_full[s], 1);
    }
    mbar_init(s_free, 4);  // the four warps of the tile that loaded S
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
  griddep_wait();  // the prologue above overlaps the previous kernel; everything below follows it
  griddep_launch_dependents();

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
                      kv0 + j * BKV, batch);
        k_issued |= 1u << st;
        k_par = (k_par & ~(1u << st)) | (ph << st);
        if (!mbar_wait(&v_empty[st], ph ^ 1, wait_limit, abort_flag, SITE_ATTN_LOAD)) { ok = false; break; }
        mbar_arrive_expect_tx(&v_full[st], TILE_BYTES);
        for (int hf = 0; hf < 2; ++hf)
          tma_load_3d(smem + OFF_V + st * TILE_BYTES + hf * HALF_BYTES, &tmV, &v_full[st], x0 + hf * 64,
                      kv0 + j * BKV, batch);
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
    // ---------------- MMA issuer: the whole warp runs the loop, one elected
    // lane issues each tcgen05 instruction ----------------
    const uint32_t sQ0 = smem_u32(smem + OFF_Q);
    bool ok = true;
    bool issued = false;
    uint32_t sfree_ph = 0;  // parity of the next s_free phase
    // Descriptors are built once: the address field of a shared-memory
    // descriptor is (address >> 4), so moving to another tile, stage or
    // 16-deep slice adds (byte offset >> 4) to the base descriptor.
    const uint64_t dQ = sdesc_sw128(sQ0, 16, 1024);
    const uint64_t dK = sdesc_sw128(smem_u32(smem + OFF_K), 16, 1024);
    const uint64_t dV = sdesc_sw128(smem_u32(smem + OFF_V), HALF_BYTES, 1024);
    const uint32_t tSacc = tmem_base + COL_S;
    auto issue_qk = [&](int t, int kst) {
      const uint64_t q = dQ + (uint64_t)((t * TILE_BYTES) >> 4);
      const uint64_t k = dK + (uint64_t)((kst * TILE_BYTES) >> 4);
#pragma unroll
      for (int kk = 0; kk < HD / 16; ++kk) {
        const uint64_t off = (uint64_t)(((kk >> 2) * HALF_BYTES + (kk & 3) * 32) >> 4);
        umma_ss_elect(tSacc, q + off, k + off, IDESC_QK, kk > 0 ? 1u : 0u);
      }
    };
    auto issue_pv = [&](int t, int vst, bool acc) {
      const uint64_t v = dV + (uint64_t)((vst * TILE_BYTES) >> 4);
      const uint32_t tO = tmem_base + COL_O + (uint32_t)(t * 128);
      const uint32_t tP = tmem_base + COL_P + (uint32_t)(t * 64);
#pragma unroll
      for (int kk = 0; kk < BKV / 16; ++kk) {
        // A: P_t in TMEM, 16 keys = 8 columns of bf16 pairs.
        // B: V MN-major; 64-d halves HALF_BYTES apart (LBO), 8-key groups 1024 B apart (SBO).
        umma_ts_elect(tO, tP + (uint32_t)(kk * 8), v + (uint64_t)((kk * 2048) >> 4), IDESC_PV,
                      (acc || kk > 0) ? 1u : 0u);
      }
    };
    // every lane waits; the warp proceeds only if all of them saw the phase
    auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, wait_limit, abort_flag, SITE_ATTN_MMA));
    };
    auto wait_sfree = [&]() -> bool {
      const bool r = wait(s_free, sfree_ph);
      sfree_ph ^= 1u;
      return r;
    };
    // prologue: S <- Q0 K_0, then (once tile 0 has loaded it) S <- Q1 K_0
    if (!wait(q_full, 0)) ok = false;
    if (ok && !wait(&k_full[0], 0)) ok = false;
    if (ok) {
      tc_fence_after();
      issue_qk(0, 0);
      umma_commit_elect(&s_full[0]);
      issued = true;
    }
    if (ok && !wait_sfree()) ok = false;
    if (ok) {
      tc_fence_after();
      issue_qk(1, 0);
      umma_commit_elect(&s_full[1]);
    }
    for (int j = 0; j < n_kv && ok; ++j) {
      const int st = j & 1;
      const uint32_t ph = (j >> 1) & 1;
      const bool has_next = j + 1 < n_kv;
      const int nst = (j + 1) & 1;
      const uint32_t nph = ((j + 1) >> 1) & 1;
      if (has_next) {  // S <- Q0 K_{j+1} once tile 1 has loaded its scores of key tile j
        if (!wait_sfree()) { ok = false; break; }
        if (!wait(&k_full[nst], nph)) { ok = false; break; }
        tc_fence_after();
        issue_qk(0, nst);
        umma_commit_elect(&s_full[0]);
      }
      if (!wait(&v_full[st], ph)) { ok = false; break; }
      if (!wait(&p_full[0], j & 1)) { ok = false; break; }
      tc_fence_after();
      issue_pv(0, st, j > 0);
      umma_commit_elect(&p_free[0]);
      if (has_next) {  // S <- Q1 K_{j+1} once tile 0 has loaded its scores of key tile j+1
        if (!wait_sfree()) { ok = false; break; }
        tc_fence_after();
        issue_qk(1, nst);
        umma_commit_elect(&s_full[1]);
      }
      if (!wait(&p_full[1], j & 1)) { ok = false; break; }
      tc_fence_after();
      issue_pv(1, st, j > 0);
      umma_commit_elect(&p_free[1]);
      umma_commit_elect(&v_empty[st]);
    }
    if (ok) {
      umma_commit_elect(&o_full[0]);
      umma_commit_elect(&o_full[1]);
    } else if (issued) {
      umma_commit_elect(drain);
      (void)mbar_wait(drain, 0, wait_limit, nullptr, SITE_ATTN_DRAIN);
    }
  } else {
    // ---------------- softmax warpgroups ----------------
    const int t = warp >> 2;          // which query tile
    const int quad = warp & 3;        // TMEM lane quadrant
    const int row = quad * 32 + lane; // query row within the tile
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t tS = tmem_base + lane_off + COL_S;
    const uint32_t tP = tmem_base + lane_off + COL_P + (uint32_t)(t * 64);
    const uint32_t tO = tmem_base + lane_off + COL_O + (uint32_t)(t * 128);
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
      // QK_1(j) is the last MMA that reads key tile j: once its scores are
      // complete, tile 1's warps release the K stage (one arrival per warp,
      // so the issuing thread spends no commit on it)
      if (t == 1 && lane == 0) mbar_arrive(&k_empty[j & 1]);
      tc_fence_after();
      // Scores in two halves: the row max of keys 0..63 runs while keys
      // 64..127 are still on their way from TMEM.
      uint32_t r[4][32];
      const int valid = kv_len - j * BKV;  // keys of this tile in this CTA's range
      auto mask = [&](int c) {
        if (valid < BKV) {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (c * 32 + i >= valid) r[c][i] = __float_as_uint(-INFINITY);
        }
      };
      // max of 32 scores: two independent chains of 3-input max
      auto cmax = [&](int c) -> float {
        float a = fmaxf(__uint_as_float(r[c][0]), __uint_as_float(r[c][1]));
        float b = fmaxf(__uint_as_float(r[c][2]), __uint_as_float(r[c][3]));
#pragma unroll
        for (int i = 4; i < 32; i += 4) {
          a = max3f(a, __uint_as_float(r[c][i]), __uint_as_float(r[c][i + 1]));
          b = max3f(b, __uint_as_float(r[c][i + 2]), __uint_as_float(r[c][i + 3]));
        }
        return fmaxf(a, b);
      };
      tmem_ld32_nowait(tS + 0u, r[0]);
      tmem_ld32_nowait(tS + 32u, r[1]);
      tmem_wait_ld();
      reg_fence32(r[0]);
      reg_fence32(r[1]);
      tmem_ld32_nowait(tS + 64u, r[2]);
      tmem_ld32_nowait(tS + 96u, r[3]);
      mask(0);
      mask(1);
      float m01 = fmaxf(cmax(0), cmax(1));
      asm volatile("" : "+f"(m01));  // computed before the wait below
      tmem_wait_ld();
      reg_fence32(r[2]);
      reg_fence32(r[3]);
      // the scores are in registers: S may take the other tile's next scores
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free);
      mask(2);
      mask(3);
      const float m_tile = fmaxf(m01, fmaxf(cmax(2), cmax(3))) * sl2;
      const bool need = m_tile > m_run + 8.0f;  // always true on the first tile
      const float m_new = need ? m_tile : m_run;
      const float alpha = need ? ex2_fast(m_run - m_new) : 1.0f;  // 0 on the first tile
      const uint64_t sl2x2 = f2_pack(sl2, sl2);
      const uint64_t negx2 = f2_pack(-m_new, -m_new);
      uint64_t sum2[2] = {0ull, 0ull};  // packed (even, odd) partial sums, two chains
      uint32_t pk[4][16];
      auto exps = [&](int c) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          // x = s * scale * log2(e) - m for the pair (2i, 2i+1): one packed FMA
          const uint64_t x = f2_fma((uint64_t)r[c][2 * i] | ((uint64_t)r[c][2 * i + 1] << 32), sl2x2, negx2);
          uint64_t pp;
          if ((i & 7) == 7) {  // an eighth of the exponentials on the FMA pipe
            pp = exp2_poly2(f2_lo(x), f2_hi(x));
          } else {
            pp = f2_pack(ex2_fast(f2_lo(x)), ex2_fast(f2_hi(x)));
          }
          sum2[i & 1] = f2_add(sum2[i & 1], pp);
          pk[c][i] = pack_bf16x2(f2_lo(pp), f2_hi(pp));
        }
      };
      // P of keys 0..63 goes to TMEM while the exponentials of keys 64..127
      // run; P_t and O_t are free once the previous PV of this tile is done
      exps(0);
      exps(1);
      if (j > 0) {
        ok = mbar_wait(&p_free[t], (j - 1) & 1, wait_limit, abort_flag, SITE_ATTN_SOFTMAX);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc_fence_after();
      }
      tmem_st16(tP + 0u, pk[0]);
      tmem_st16(tP + 16u, pk[1]);
      exps(2);
      exps(3);
      const uint64_t st2 = f2_add(sum2[0], sum2[1]);
      l_run = l_run * alpha + (f2_lo(st2) + f2_hi(st2));
      tmem_st16(tP + 32u, pk[2]);
      tmem_st16(tP + 48u, pk[3]);
      // Rescale O_t when any row of this warp raised its max
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
      const bool live = qi < p.Sq;
      bf16* orow = p.o + split * p.o_split_stride + ((int64_t)batch * p.Sq + qi) * p.ldo + head * HD;
      const int64_t li = split * p.lse_split_stride + ((int64_t)batch * p.H + head) * p.Sq + qi;
      const float lse_cur = (m_run + __log2f(l_run)) * 0.6931471805599453f;  // natural log
      // o = w_prev o_prev + w_cur (O / l): w_prev = 0, w_cur = 1 unless accumulating
      float w_prev = 0.0f, w_cur = 1.0f / l_run, lse_new = lse_cur;
      if (p.accumulate && live) {
        const float lse_prev = p.lse[li];  // -inf: nothing accumulated yet
        const float mx = fmaxf(lse_prev, lse_cur);
        const float ep = __expf(lse_prev - mx), ec = __expf(lse_cur - mx);
        const float inv = 1.0f / (ep + ec);
        lse_new = mx + __logf(ep + ec);
        w_prev = ep * inv;
        w_cur *= ec * inv;
      }
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(tO + (uint32_t)(c * 32), r);
        if (live) {
          uint4* dp = reinterpret_cast<uint4*>(orow + c * 32);
          float pv[32];
          if (p.accumulate) {  // this thread's own row: read before it is written
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint4 u = dp[q];
              pv[8 * q + 0] = bf16_lo(u.x); pv[8 * q + 1] = bf16_hi(u.x);
              pv[8 * q + 2] = bf16_lo(u.y); pv[8 * q + 3] = bf16_hi(u.y);
              pv[8 * q + 4] = bf16_lo(u.z); pv[8 * q + 5] = bf16_hi(u.z);
              pv[8 * q + 6] = bf16_lo(u.w); pv[8 * q + 7] = bf16_hi(u.w);
            }
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) pv[i] = 0.0f;
          }
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float o8[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) o8[i] = fmaf(__uint_as_float(r[8 * q + i]), w_cur, w_prev * pv[8 * q + i]);
            uint4 w;
            w.x = pack_bf16x2(o8[0], o8[1]);
            w.y = pack_bf16x2(o8[2], o8[3]);
            w.z = pack_bf16x2(o8[4], o8[5]);
            w.w = pack_bf16x2(o8[6], o8[7]);
            dp[q] = w;
          }
        }
      }
      if (p.lse != nullptr && live) p.lse[li] = lse_new;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 9) tmem_dealloc(tmem_base, TMEM_COLS);
}

}  // namespace attn
}  // namespace dit

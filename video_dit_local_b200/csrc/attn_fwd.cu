// Attention forward on tcgen05 tensor cores, one kernel for both branches:
//  - FWD_STA: sliding-tile attention ("Fast Video Generation with Sliding Tile
//    Attention", abstract).  The query block lies inside one query tile, or
//    (PAIR instance, tile volumes an odd multiple of 64 rows) straddles two
//    w-adjacent tiles (PairPlan, common.cuh); its key stream is the box of
//    kept tiles (for a straddling block the union of the two windows),
//    computed here from the tile coordinate, so masked tiles are never loaded.
//  - FWD_GLOBAL: every query attends to all pooled keys ("UltraGen ..." §4.2),
//    with an optional blend epilogue O = g*O_local + (1-g)*O_global (§4.1).
//
// CTA = 128 query rows, 11 warps:
//   warps 0-3  softmax group 0 (even key blocks), warps 4-7 softmax group 1
//   (odd key blocks); each group owns one S accumulator and one O
//   accumulator in TMEM (S0 cols 0-127, S1 128-255, O0 256+, O1 384+), and
//   the two partial results are merged in the epilogue;
//   warp 8 loads Q and K, warp 9 loads V (TMA, 128-byte swizzle, each CTA
//   its own tiles); warp 10 issues the MMAs and owns the TMEM allocation.
// P is written back over its own S columns as bf16 and read by the P*V MMA
// straight from TMEM.  The running max is only moved (and O rescaled) when a
// row's max grows by more than 2^8; otherwise P may reach 2^8, which bf16 and
// the fp32 accumulators carry without loss of relative precision.
//
// FP8 variant (inference): F8 takes Q and K as e4m3 bytes (Q*K^T on the
// f8f6f4 tensor path, the dequantisation folded into the softmax constant);
// F8V also takes V as e4m3 bytes and rounds P to e4m3 (packed four to a TMEM
// column), so P*V is four K = 32 instructions per key block instead of
// eight; V's scale is applied in the epilogue.
#include "fwd_common.cuh"

namespace vattn {

namespace fwd {

constexpr int NTHREADS = 352;
constexpr int WARP_QK_LOAD = 8;
constexpr int WARP_V_LOAD = 9;
constexpr int WARP_MMA = 10;
constexpr int NK = 3;  // K ring stages
constexpr int NV = 2;  // V ring stages
constexpr float RESCALE_LOG2_THRESHOLD = 8.0f;
// Bit b set: the exponentials of the b-th group of 16 columns (of 8) run on
// the FMA pipe (exp2_poly) instead of the MUFU unit, shortening the MUFU part
// of a softmax phase at the cost of FMA-pipe instructions.
#ifndef VATTN_FWD_POLY_MASK
#define VATTN_FWD_POLY_MASK 0x00
#endif
constexpr int POLY_MASK = VATTN_FWD_POLY_MASK;

// F8: Q and K are e4m3 bytes (one 128-byte box per row at d = 128); F8V: V
// too (P*V on e4m3 operands, P rounded to e4m3).
template <int D, bool F8 = false, bool F8V = false>
struct Smem {
  static constexpr int CHUNKS = D / 64;                 // 64-column (128-byte) swizzle boxes
  static constexpr int QK_CHUNKS = F8 ? D / 128 : CHUNKS;   // 128-byte boxes per Q / K row
  static constexpr int QK_ELEMS = F8 ? 128 : 64;            // elements per box row
  static constexpr int QK_BYTES = QK_CHUNKS * 128 * 128;    // 128 rows of Q or K
  static constexpr int V_CHUNKS = F8V ? D / 128 : CHUNKS;   // 128-byte boxes per V row
  static constexpr int V_ELEMS = F8V ? 128 : 64;
  static constexpr int V_BYTES = V_CHUNKS * 128 * 128;      // 128 rows of V
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + QK_BYTES;
  static constexpr int OFF_V = OFF_K + NK * QK_BYTES;
  static constexpr int OFF_BAR = OFF_V + NV * V_BYTES;
  static constexpr int NBAR = 1 + 2 * NK + 2 * NV + 2 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int OFF_XCH = OFF_MISC + 16;
  static constexpr int TOTAL = OFF_XCH + 2 * 128 * 2 * 4;
  static constexpr int ALLOC = TOTAL + 1024;
};

// PAIR: query blocks of adjacent tiles paired along w (tile volumes an odd
// multiple of BM/2); see QueryBlock.
template <int D, bool F8 = false, bool F8V = false, bool PAIR = false>
__global__ void __launch_bounds__(NTHREADS, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const Params p) {
  static_assert(!F8V || (F8 && D == 128), "e4m3 P*V comes with e4m3 Q*K^T at d = 128");
  using L = Smem<D, F8, F8V>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  // qk_done[j % NK] completes when Q*K_j^T is done: it tells softmax group
  // j & 1 that S_j is in TMEM and the K loader that stage j % NK is free.  Both
  // wait for a phase before the barrier can complete the next one (block j+3
  // needs K_{j+3}, loaded after the loader's wait, and its Q*K^T is issued
  // after P_j, produced after the group's wait), so one commit serves both.
  uint64_t* qk_done = k_full + NK;
  uint64_t* v_full = qk_done + NK;
  uint64_t* v_empty = v_full + NV;
  uint64_t* p_full = v_empty + NV;
  uint64_t* o_final = p_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);
  float2* xch = reinterpret_cast<float2*>(smem + L::OFF_XCH);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  const int qblk = blockIdx.x;
  WaitCtx wc;
  wc.abort_flag = abort_flag;
  wc.timeout_ns = p.ctl.timeout_ns;
  wc.err_word = p.ctl.err_word;

  // query block -> rows and key stream
  const QueryBlock qb = query_block<PAIR>(p, qblk);
  const int q_tile = qb.tile, q_row0 = qb.row0, q_valid = qb.valid, sub = qb.sub;
  const Stream st = make_block_stream<PAIR>(p, qb);
  const int L_total = st.length();
  const int nblk = (L_total + BN - 1) / BN;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < NK; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&qk_done[i], 1);
    }
    for (int i = 0; i < NV; ++i) {
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&p_full[i], 4);  // one arrival per softmax warp
    }
    mbar_init(o_final, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == WARP_MMA) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (warp == WARP_QK_LOAD && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  constexpr uint32_t BOX_BYTES = 128 * 128;   // one 128-row x 128-byte box
  const uint32_t sub_bytes = (uint32_t)p.G * 128;
  const int subs = BN / p.G;

  if (warp == WARP_QK_LOAD) {
    if (lane == 0) {
      int issued_k = 0;
      KeyCursor kc = key_cursor(p, st, L_total);  // e4m3 instance (see KeyCursor)
      const int tiles_per_run = p.mode == FWD_STA ? st.run_len / p.g.s : 1;
      if (!dcheck(query_block_ok(p, q_row0, q_valid), p.ctl.err_word)) *abort_flag = 1;
      if (!(p.ctl.debug_flags & 1) && !*abort_flag) {
        mbar_arrive_expect_tx(q_full, L::QK_BYTES);
        if (p.raster) {
          const DevGeom& g = p.g;
          const int at = q_tile / (g.Nh * g.Nw), ah = (q_tile / g.Nw) % g.Nh, aw = q_tile % g.Nw;
          const int t0 = at * g.tt + sub * BM / (g.th * g.tw);
          for (int c = 0; c < L::QK_CHUNKS; ++c)
            tma_load_5d(smem + L::OFF_Q + c * BOX_BYTES, &tm_q, q_full, c * L::QK_ELEMS, aw * g.tw, ah * g.th, t0, bh);
        } else {
          for (int c = 0; c < L::QK_CHUNKS; ++c)
            tma_load_3d(smem + L::OFF_Q + c * BOX_BYTES, &tm_q, q_full, c * L::QK_ELEMS, q_row0, bh);
        }
      }
      for (int j = 0; j < nblk; ++j) {
        const int s = j % NK, r = j / NK;
        if (!mbar_wait(&qk_done[s], (r & 1) ^ 1, wc)) break;
        if (!dcheck(key_block_ok(p, st, j, L_total), p.ctl.err_word)) {
          *abort_flag = 1;
          break;
        }
        mbar_arrive_expect_tx(&k_full[s], L::QK_BYTES);
        uint8_t* dst = smem + L::OFF_K + s * L::QK_BYTES;
        for (int u = 0; u < subs; ++u) {
          const int v = j * BN + u * p.G;
          if (!F8 && p.raster) {
            int x, y, t;
            stream_box(p, st, v, L_total, &x, &y, &t);
            for (int c = 0; c < L::QK_CHUNKS; ++c)
              tma_load_5d(dst + c * BOX_BYTES + u * sub_bytes, &tm_k, &k_full[s], c * L::QK_ELEMS, x, y, t, bh);
          } else {
            int row;  // past the end: row Nk, zero fill
            if constexpr (F8) {
              row = cursor_row(p, st, kc);
              cursor_next(p, st, kc, tiles_per_run);
            } else {
              row = v < L_total ? stream_row(p, st, v) : p.Nk;
            }
            for (int c = 0; c < L::QK_CHUNKS; ++c)
              tma_load_3d(dst + c * BOX_BYTES + u * sub_bytes, &tm_k, &k_full[s], c * L::QK_ELEMS, row, bh);
          }
        }
        ++issued_k;
      }
      {  // every issued load has landed before the CTA can exit (a no-op unless aborted)
        for (int j = issued_k - NK < 0 ? 0 : issued_k - NK; j < issued_k; ++j)
          mbar_wait_drain(&k_full[j % NK], (j / NK) & 1, wc);
      }
    }
  } else if (warp == WARP_V_LOAD) {
    if (lane == 0) {
      int issued_v = 0;
      KeyCursor vc = key_cursor(p, st, L_total);
      const int tiles_per_run = p.mode == FWD_STA ? st.run_len / p.g.s : 1;
      for (int j = 0; j < nblk; ++j) {
        const int s = j % NV, r = j / NV;
        if (!mbar_wait(&v_empty[s], (r & 1) ^ 1, wc)) break;
        if (!dcheck(key_block_ok(p, st, j, L_total), p.ctl.err_word)) {
          *abort_flag = 1;
          break;
        }
        mbar_arrive_expect_tx(&v_full[s], L::V_BYTES);
        uint8_t* dst = smem + L::OFF_V + s * L::V_BYTES;
        for (int u = 0; u < subs; ++u) {
          const int v = j * BN + u * p.G;
          if (!F8 && p.raster) {
            int x, y, t;
            stream_box(p, st, v, L_total, &x, &y, &t);
            for (int c = 0; c < L::V_CHUNKS; ++c)
              tma_load_5d(dst + c * BOX_BYTES + u * sub_bytes, &tm_v, &v_full[s], c * L::V_ELEMS, x, y, t, bh);
          } else {
            int row;
            if constexpr (F8) {
              row = cursor_row(p, st, vc);
              cursor_next(p, st, vc, tiles_per_run);
            } else {
              row = v < L_total ? stream_row(p, st, v) : p.Nk;
            }
            for (int c = 0; c < L::V_CHUNKS; ++c)
              tma_load_3d(dst + c * BOX_BYTES + u * sub_bytes, &tm_v, &v_full[s], c * L::V_ELEMS, row, bh);
          }
        }
        ++issued_v;
      }
      {
        for (int j = issued_v - NV < 0 ? 0 : issued_v - NV; j < issued_v; ++j)
          mbar_wait_drain(&v_full[j % NV], (j / NV) & 1, wc);
      }
    }
  } else if (warp == WARP_MMA) {
    if (lane == 0) {
      constexpr uint32_t IDESC_QK = idesc_bf16_f32(BM, BN, 0, 0);
      constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, D, 0, 1);
      const uint32_t q_base = smem_u32(smem + L::OFF_Q);
      const uint32_t k_base = smem_u32(smem + L::OFF_K);
      const uint32_t v_base = smem_u32(smem + L::OFF_V);
      bool ok = mbar_wait(q_full, 0, wc);
      auto issue_qk = [&](int j) -> bool {
        const int s = j % NK;
        if (!mbar_wait(&k_full[s], (j / NK) & 1, wc)) return false;
        tc_fence_after();
        const uint32_t kb = k_base + s * L::QK_BYTES;
        const uint32_t d_tmem = tmem + (uint32_t)((j & 1) * 128);
        // four 32-byte K-steps per 128-byte box: 16 bf16 or 32 e4m3 elements each
#pragma unroll
        for (int kk = 0; kk < L::QK_CHUNKS * 4; ++kk) {
          const uint32_t off = (kk >> 2) * BOX_BYTES + (kk & 3) * 32;
          if constexpr (F8)
            mma_ss_e4m3(d_tmem, smem_desc_sw128(q_base + off, 16, 1024), smem_desc_sw128(kb + off, 16, 1024),
                        idesc_e4m3_f32(BM, BN), kk > 0);
          else
            mma_ss(d_tmem, smem_desc_sw128(q_base + off, 16, 1024), smem_desc_sw128(kb + off, 16, 1024), IDESC_QK,
                   kk > 0);
        }
        tc_commit(&qk_done[s]);
        return true;
      };
      if (ok) ok = issue_qk(0);
      if (ok && nblk > 1) ok = issue_qk(1);
      for (int j = 0; ok && j < nblk; ++j) {
        const int w = j & 1;
        if (!mbar_wait(&p_full[w], (j >> 1) & 1, wc)) break;
        const int s = j % NV;
        if (!mbar_wait(&v_full[s], (j / NV) & 1, wc)) break;
        tc_fence_after();
        const uint32_t vb = v_base + s * L::V_BYTES;
        const uint32_t o_tmem = tmem + 256 + (uint32_t)(w * 128);
        const uint32_t p_tmem = tmem + (uint32_t)(w * 128);
        if constexpr (F8V) {
          // e4m3: four K = 32 steps; A = P packed four to a TMEM column; B = V
          // block (keys x d, one 128-byte row per key), MN-major, SBO = next 8 keys
#pragma unroll
          for (int kk = 0; kk < BN / 32; ++kk)
            mma_ts_e4m3(o_tmem, p_tmem + kk * 8, smem_desc_sw128(vb + kk * 4096, BOX_BYTES, 1024),
                        idesc_e4m3_f32_bmn(BM, D), (j >= 2 || kk > 0) ? 1u : 0u);
        } else {
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            // B = V block (keys x d), MN-major: LBO = next 64-column box, SBO = next 8 keys
            mma_ts(o_tmem, p_tmem + kk * 8, smem_desc_sw128(vb + kk * 2048, BOX_BYTES, 1024), IDESC_PV,
                   (j >= 2 || kk > 0) ? 1u : 0u);
          }
        }
        tc_commit(&v_empty[s]);
        if (j + 2 < nblk) ok = issue_qk(j + 2);
      }
      tc_commit(o_final);
      // every MMA this thread issued must be finished before TMEM is freed
      mbar_wait_drain(o_final, 0, wc);
    }
  } else {
    // ---------------- softmax groups ----------------
    const int w = warp >> 2;            // group 0: warps 0-3, group 1: warps 4-7
    const int quad = warp & 3;          // TMEM lane quarter
    const int row = quad * 32 + lane;   // query row within the block
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    const uint32_t tS = tmem + lane_addr + (uint32_t)(w * 128);
    const uint32_t tO = tmem + lane_addr + 256u + (uint32_t)(w * 128);
    float c2 = p.scale_log2;
    if constexpr (F8) {  // S = bytes(Q) bytes(K)^T * (absmax_Q / 448) * (absmax_K / 448)
      const float aq = __int_as_float(p.qk_amax[2 * bh]), ak = __int_as_float(p.qk_amax[2 * bh + 1]);
      c2 *= (aq > 0.f ? aq / 448.f : 1.f) * (ak > 0.f ? ak / 448.f : 1.f);
    }
    // e4m3 P: the running max moves when a row's max grows by more than 2^2,
    // so P <= 2^2 and P * 2^6 <= 2^8 < 448 (the largest e4m3); the factor 2^6
    // (folded into the exponent) keeps small probabilities out of e4m3's
    // subnormal range and cancels against the row sum, accumulated in the
    // same units.
    constexpr float THRESH = F8V ? 2.0f : RESCALE_LOG2_THRESHOLD;
    constexpr float PSHIFT = F8V ? 6.0f : 0.0f;
    float m_ref = -INFINITY, l_sum = 0.f;
    int qs = w;          // qk_done stage of this group's next block (j % NK) ...
    uint32_t qph = 0;    // ... and its phase parity ((j / NK) & 1)
    bool ok = true;
    int o_blk = (F8 && PAIR && st.rot) ? (w * BN) % st.run_len : 0;  // run offset of this group's next block
    for (int i = 0;; ++i) {
      const int j = 2 * i + w;
      if (j >= nblk) break;
      ok = mbar_wait(&qk_done[qs], qph, wc);
      qs += 2;  // next block of this group: j + 2
      if (qs >= NK) {
        qs -= NK;
        qph ^= 1u;
      }
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[4][32];
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) tmem_ld32(tS + q4 * 32, sr[q4]);
      tmem_wait_ld();
      const int valid = L_total - j * BN;
      if (valid < BN) {
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4)
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (q4 * 32 + c >= valid) sr[q4][c] = __float_as_uint(-INFINITY);
      }
      if (PAIR && st.rot) {
        // straddling block over windows one tile apart: the first tile's rows
        // (quads 0, 1) see run tiles 0 .. ew-1 (w0+1 .. w0+ew), the second's
        // (quads 2, 3) run tiles 0 .. ew-2 and ew (w0+1 .. w0+ew-1, then w0);
        // 32-column groups never cross a tile (s is a multiple of 64)
        const int x0 = straddle_excluded_start(p.g.s, st.ew, quad >> 1);  // excluded run offsets [x0, x0 + s)
        int o;
        if constexpr (F8) {  // no division in the e4m3 kernel (see KeyCursor)
          o = o_blk;
          o_blk += 2 * BN;  // this group's next block
          while (o_blk >= st.run_len) o_blk -= st.run_len;
        } else {
          o = (j * BN) % st.run_len;
        }
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          int oq = o + q4 * 32;
          if (oq >= st.run_len) oq -= st.run_len;
          if ((unsigned)(oq - x0) < (unsigned)p.g.s) {
#pragma unroll
            for (int c = 0; c < 32; ++c) sr[q4][c] = __float_as_uint(-INFINITY);
          }
        }
      }
      // row max: four independent chains of three-input max
      float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4)
#pragma unroll
        for (int c = 0; c < 32; c += 2)
          m4[(c >> 1) & 3] = fmax3(m4[(c >> 1) & 3], __uint_as_float(sr[q4][c]), __uint_as_float(sr[q4][c + 1]));
      const float mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
      const float mx2 = mx * c2;
      bool need = false;
      if (i == 0) {
        m_ref = mx2;
      } else if (mx2 > m_ref + THRESH) {
        need = true;
      }
      float alpha = 1.f;
      if (need) {
        alpha = ex2(m_ref - mx2);
        m_ref = mx2;
        l_sum *= alpha;
      }
      // P = 2^(S*scale*log2(e) - m (+ PSHIFT)) two lanes at a time (packed fp32x2)
      const float2 c2x2 = make_float2(c2, c2), negm2 = make_float2(PSHIFT - m_ref, PSHIFT - m_ref);
      float2 s2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        uint32_t pk[16];
        uint32_t p8[8];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const float2 x = ffma2(make_float2(__uint_as_float(sr[q4][2 * c]), __uint_as_float(sr[q4][2 * c + 1])),
                                 c2x2, negm2);
          float2 pp;
          if ((POLY_MASK >> (q4 * 2 + (c >> 3))) & 1) {  // FMA-pipe exponentials for this group of 16
            pp.x = exp2_poly(x.x);
            pp.y = exp2_poly(x.y);
          } else {
            pp.x = ex2(x.x);
            pp.y = ex2(x.y);
          }
          s2[c & 1] = fadd2(s2[c & 1], pp);
          if constexpr (F8V) {
            const uint32_t h = pack_e4m3x2(pp.x, pp.y);
            p8[c >> 1] = (c & 1) ? (p8[c >> 1] | (h << 16)) : h;
          } else {
            pk[c] = pack_bf16(pp.x, pp.y);
          }
        }
        if constexpr (F8V)
          tmem_st8(tS + q4 * 8, p8);
        else
          tmem_st16(tS + q4 * 16, pk);
      }
      l_sum += (s2[0].x + s2[0].y) + (s2[1].x + s2[1].y);
      if (__any_sync(0xffffffffu, need)) {
        // O of this group is quiescent: the commit that signalled this S also
        // covers the previous P*V into it, and the next one waits for p_full.
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t o[32];
          tmem_ld32(tO + c0, o);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
          tmem_st32(tO + c0, o);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[w]);
    }
    // ---------------- epilogue ----------------
    if (ok && !*abort_flag) ok = mbar_wait(o_final, 0, wc);
    ok = __all_sync(0xffffffffu, ok);
    tc_fence_after();
    xch[w * 128 + row] = make_float2(m_ref, l_sum);
    named_bar_sync(1, 256);
    if (ok && !*abort_flag) {
      const float2 other = xch[(1 - w) * 128 + row];
      const float m = fmaxf(m_ref, other.x);
      const float a_self = ex2(m_ref - m), a_other = ex2(other.x - m);
      const float l = l_sum * a_self + other.y * a_other;
      float inv_l = 1.f / l;
      if constexpr (F8V) {  // O = P V with V = bytes(V) * absmax_V / 448
        const float av = __int_as_float(p.v_amax[bh]);
        inv_l *= av > 0.f ? av / 448.f : 1.f;
      }
      const float a0 = (w == 0 ? a_self : a_other) * inv_l;
      const float a1 = (w == 0 ? a_other : a_self) * inv_l;
      const bool have1 = nblk >= 2;
      bool row_ok = row < q_valid;
      size_t grow = (size_t)bh * p.g.N + (size_t)(q_row0 + row);
      if (p.raster) {  // tile-major row -> raster token
        const DevGeom& g = p.g;
        const int at = q_tile / (g.Nh * g.Nw), ah = (q_tile / g.Nw) % g.Nh, aw = q_tile % g.Nw;
        const int lr = sub * BM + row;
        const int lt = lr / (g.th * g.tw), lh = (lr / g.tw) % g.th, lw = lr % g.tw;
        grow = (size_t)bh * g.N + ((size_t)(at * g.tt + lt) * g.H + (ah * g.th + lh)) * g.W + (aw * g.tw + lw);
      }
      if (row_ok && !dcheck(out_row_ok(p, bh, grow), p.ctl.err_word)) row_ok = false;
      // hierarchical merge: one softmax over the fine keys (O_f, LSE_f given)
      // and this kernel's coarse keys, in log2 units
      float wf = 0.f, wc = 1.f, lse2_out = m - PSHIFT + __log2f(l);
      if (p.merge_o && row_ok) {
        const float lf2 = p.merge_lse[grow] * 1.4426950408889634f;
        const float mm = fmaxf(lf2, lse2_out);
        wf = ex2(lf2 - mm);
        wc = ex2(lse2_out - mm);
        const float inv = 1.f / (wf + wc);
        lse2_out = mm + __log2f(wf + wc);
        wf *= inv;
        wc *= inv;
      }
      const uint32_t tO0 = tmem + lane_addr + 256u, tO1 = tmem + lane_addr + 384u;
      float gh = 0.f;
      if (p.blend_out) gh = p.gvec[bh % p.g.heads];
#pragma unroll
      for (int c0 = (w * D) / 2; c0 < ((w + 1) * D) / 2; c0 += 32) {
        uint32_t x0[32], x1[32];
        tmem_ld32(tO0 + c0, x0);
        if (have1) tmem_ld32(tO1 + c0, x1);
        tmem_wait_ld();
        float* o = reinterpret_cast<float*>(x0);
#pragma unroll
        for (int c = 0; c < 32; ++c)
          o[c] = __uint_as_float(x0[c]) * a0 + (have1 ? __uint_as_float(x1[c]) * a1 : 0.f);
        if (row_ok && p.merge_o) {
          const uint4* src = reinterpret_cast<const uint4*>(p.merge_o + grow * D + c0);
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4) {
            const uint4 of = src[v4];
            const uint32_t w4[4] = {of.x, of.y, of.z, of.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              o[8 * v4 + 2 * e] = wf * bf16lo(w4[e]) + wc * o[8 * v4 + 2 * e];
              o[8 * v4 + 2 * e + 1] = wf * bf16hi(w4[e]) + wc * o[8 * v4 + 2 * e + 1];
            }
          }
        }
        if (row_ok) {
          if (p.o) {
            uint4* dst = reinterpret_cast<uint4*>(p.o + grow * D + c0);
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4)
              dst[v4] = make_uint4(pack_bf16(o[8 * v4 + 0], o[8 * v4 + 1]), pack_bf16(o[8 * v4 + 2], o[8 * v4 + 3]),
                                   pack_bf16(o[8 * v4 + 4], o[8 * v4 + 5]), pack_bf16(o[8 * v4 + 6], o[8 * v4 + 7]));
          }
          if (p.blend_out) {
            const uint4* src = reinterpret_cast<const uint4*>(p.o_local + grow * D + c0);
            uint4* dst = reinterpret_cast<uint4*>(p.blend_out + grow * D + c0);
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4) {
              const uint4 ol = src[v4];
              const uint32_t w4[4] = {ol.x, ol.y, ol.z, ol.w};
              uint32_t r4[4];
#pragma unroll
              for (int e = 0; e < 4; ++e)
                r4[e] = pack_bf16(gh * bf16lo(w4[e]) + (1.f - gh) * o[8 * v4 + 2 * e],
                                  gh * bf16hi(w4[e]) + (1.f - gh) * o[8 * v4 + 2 * e + 1]);
              dst[v4] = make_uint4(r4[0], r4[1], r4[2], r4[3]);
            }
          }
        }
      }
      if (w == 0 && row_ok && p.lse) p.lse[grow] = lse2_out * 0.69314718055994531f;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace fwd

template <int D, bool F8, bool F8V, bool PAIR>
static cudaError_t launch_fwd1(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                               const fwd::Params& p, dim3 grid, cudaStream_t st) {
  using namespace fwd;
  auto kernel = attn_fwd_kernel<D, F8, F8V, PAIR>;
  constexpr int smem = Smem<D, F8, F8V>::ALLOC;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  kernel<<<grid, NTHREADS, smem, st>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

template <int D, bool F8 = false>
static cudaError_t launch_fwd_d(const DevGeom& g, FwdMode mode, const FwdArgs& a, cudaStream_t st) {
  using namespace fwd;
  Params p;
  p.g = g;
  p.mode = mode;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.o = (__nv_bfloat16*)a.o;
  p.lse = a.lse;
  p.o_local = (const __nv_bfloat16*)a.o_local;
  p.gvec = a.g;
  p.blend_out = a.o_local ? (__nv_bfloat16*)a.blend_out : nullptr;
  p.ctl = current_ctl();
  p.kNt = g.Nt;
  p.kNh = g.Nh;
  p.kNw = g.Nw;
  p.cft = p.cfh = p.cfw = 1;
  p.merge_o = nullptr;
  p.merge_lse = nullptr;
  p.qk_amax = a.qk_amax;
  p.v_amax = a.v_amax;
  p.raster = a.raster ? 1 : 0;
  int qblocks;
  bool pair = false;
  if (mode == FWD_STA) {
    int G = 1;
    while (G < BN && g.s % (G * 2) == 0) G *= 2;
    p.G = G;
    p.q_blocks_per_tile = (g.s + BM - 1) / BM;
    p.Nk = g.N;
    if (a.kgeom) {  // hierarchical: coarse tiles of the medium-pooled grid (same tile volume)
      p.kNt = a.kgeom->Nt;
      p.kNh = a.kgeom->Nh;
      p.kNw = a.kgeom->Nw;
      p.cft = a.cf[0];
      p.cfh = a.cf[1];
      p.cfw = a.cf[2];
      p.Nk = a.kgeom->N;
      p.merge_o = (const __nv_bfloat16*)a.merge_o;
      p.merge_lse = a.merge_lse;
    }
    qblocks = g.n_tiles * p.q_blocks_per_tile;
    // tiles of an odd multiple of BM/2 rows: pair adjacent tiles along w so
    // that no query block is half empty (tile-major rows; sliding windows of
    // at least two tiles along w, so a straddling block's first key tile is in
    // both windows)
    p.pair = make_pair_plan(g, p.kNw, !p.raster);
    if (pair_plan_active(p.pair)) {
      qblocks = (int)pair_plan_blocks(g, p.pair);
      pair = true;
    }
  } else {
    p.G = BN;
    p.q_blocks_per_tile = 1;
    p.pair = make_pair_plan(g, g.Nw, false);
    p.Nk = g.Np;
    qblocks = (g.N + BM - 1) / BM;
  }
  const long long bh = (long long)g.B * g.heads;
  if (qblocks == 0 || bh == 0) return cudaSuccess;
  CUtensorMap tq, tk, tv;
  const char* err = nullptr;
  bool maps_ok;
  const bool f8v = F8 && a.v_amax != nullptr;  // e4m3 P*V: V bytes
  if (p.raster) {  // 5-D raster maps: boxes of whole t-slices of one tile
    const int slice = g.th * g.tw;
    if (F8 || mode != FWD_STA || a.kgeom || BM % slice || p.G % slice) return cudaErrorInvalidValue;
    maps_ok = make_tmap_raster(&tq, a.q, D, g, bh, BM / slice, &err) &&
              make_tmap_raster(&tk, a.k, D, g, bh, p.G / slice, &err) &&
              make_tmap_raster(&tv, a.v, D, g, bh, p.G / slice, &err);
  } else if constexpr (F8) {
    maps_ok = make_tmap_rows_u8(&tq, a.q, D, g.N, bh, BM, &err) && make_tmap_rows_u8(&tk, a.k, D, p.Nk, bh, p.G, &err) &&
              (f8v ? make_tmap_rows_u8(&tv, a.v, D, p.Nk, bh, p.G, &err)
                   : make_tmap_rows(&tv, a.v, D, p.Nk, bh, p.G, &err));
  } else {
    maps_ok = make_tmap_rows(&tq, a.q, D, g.N, bh, BM, &err) && make_tmap_rows(&tk, a.k, D, p.Nk, bh, p.G, &err) &&
              make_tmap_rows(&tv, a.v, D, p.Nk, bh, p.G, &err);
  }
  if (!maps_ok) return cudaErrorInvalidValue;
  const dim3 grid(qblocks, (unsigned)bh);
  if constexpr (F8) {
    if (!f8v) return cudaErrorInvalidValue;  // the FP8 forward takes e4m3 V as well
    if (pair) return launch_fwd1<D, true, true, true>(tq, tk, tv, p, grid, st);
    return launch_fwd1<D, true, true, false>(tq, tk, tv, p, grid, st);
  } else {
    if (pair) return launch_fwd1<D, false, false, true>(tq, tk, tv, p, grid, st);
    return launch_fwd1<D, false, false, false>(tq, tk, tv, p, grid, st);
  }
}

__global__ void exp2_poly_kernel(const float* __restrict__ x, float* __restrict__ y, long long n) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
    y[i] = exp2_poly(x[i]);
}

cudaError_t launch_exp2_poly(const float* x, float* y, long long n, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  long long blocks = (n + 255) / 256;
  if (blocks > 4096) blocks = 4096;
  exp2_poly_kernel<<<(int)blocks, 256, 0, st>>>(x, y, n);
  return cudaGetLastError();
}

cudaError_t launch_attn_fwd(const DevGeom& g, FwdMode mode, const FwdArgs& a, cudaStream_t st) {
  if (a.v_amax && !a.qk_amax) return cudaErrorInvalidValue;  // e4m3 P*V comes with e4m3 Q*K^T
  if (a.qk_amax) {  // e4m3 Q*K^T: sliding tile or global (+ blend), d = 128
    if (g.d != 128 || a.kgeom || a.raster) return cudaErrorInvalidValue;
    return launch_fwd_d<128, true>(g, mode, a, st);
  }
  if (g.d == 128) return launch_fwd_d<128>(g, mode, a, st);
  if (g.d == 64) return launch_fwd_d<64>(g, mode, a, st);
  return cudaErrorInvalidValue;
}

}  // namespace vattn

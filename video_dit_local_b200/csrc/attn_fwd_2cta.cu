// Attention forward with two co-resident CTAs per SM, each with its own
// tcgen05 issuing thread.  Same modes and results as attn_fwd.cu (sliding
// tile, global with the blend epilogue, hierarchical merge, raster boxes,
// e4m3 Q*K^T); only the work split differs.
//
// Why two CTAs: a single issuing thread leaves the tensor pipe idle while it
// waits on barriers and commits between groups of MMAs (the pipe queues only
// about one MMA ahead of the executing one).  Two CTAs on one SM issue
// independently, so one CTA's MMAs fill the other's pauses.  Each CTA fits in
// half of the SM: 256 TMEM columns (S 0-127, O 128+), about 100 KB of shared
// memory, 128 registers per thread at launch.
//
// CTA = 128 query rows, 8 warps (two warpgroups):
//   warps 0-3  softmax (TMEM lane quarter = warp), 192 registers each after
//              setmaxnreg;
//   warp 4     loads Q and K, warp 5 loads V (TMA, 128-byte swizzle, no
//              multicast); warp 6 issues the MMAs and owns the TMEM
//              allocation; warp 7 idles; 64 registers each.
// Per 128-key block j: S = Q K_j^T into S; the softmax writes P_j (bf16) over
// its own S columns; O += P_j V_j reads P from TMEM; then S = Q K_{j+1}^T is
// issued behind it (tensor-pipe order keeps P_j intact until it is read).
// The running max only moves (and O is rescaled) when a row's max grows by
// more than 2^8.  A fraction of the exponentials run on the FMA pipe
// (exp2_poly) so the MUFU unit does not limit the pair of CTAs.
#include <algorithm>

#include "fwd_common.cuh"

namespace vattn {
namespace fwd2 {

using fwd::BM;
using fwd::BN;
using fwd::Params;
using fwd::Stream;

constexpr int NTHREADS = 256;
constexpr int WARP_QK_LOAD = 4;
constexpr int WARP_V_LOAD = 5;
constexpr int WARP_MMA = 6;
constexpr int TMEM_COLS = 256;
constexpr uint32_t S_COL = 0, O_COL = 128;
constexpr float RESCALE_LOG2_THRESHOLD = 8.0f;
// Bit c set: the exponentials of 32-column chunk c (of 4) run on the FMA pipe.
#ifndef VATTN_FWD2_POLY_MASK
#define VATTN_FWD2_POLY_MASK 0x8
#endif
constexpr int POLY_MASK = VATTN_FWD2_POLY_MASK;
// Register budgets after setmaxnreg: 128 x 192 + 128 x 64 = 256 x 128, the
// registers the CTA is launched with.
constexpr uint32_t REGS_SOFTMAX = 192, REGS_OTHER = 64;
static_assert(128 * REGS_SOFTMAX + 128 * REGS_OTHER <= NTHREADS * 128, "register split exceeds the launch budget");

// Shared memory budget per CTA: at most (228 KB - 2 x 1 KB reserved) / 2.
// F8: Q and K are e4m3 bytes; F8V: V is e4m3 bytes too (one 128-byte box per
// row at d = 128).
template <int D, bool F8, bool F8V = false>
struct Smem2 {
  static constexpr int CHUNKS = D / 64;                    // 64-column (128-byte) swizzle boxes
  static constexpr int QK_CHUNKS = F8 ? D / 128 : CHUNKS;  // 128-byte boxes per Q / K row
  static constexpr int QK_ELEMS = F8 ? 128 : 64;           // elements per box row
  static constexpr int QK_BYTES = QK_CHUNKS * 128 * 128;   // 128 rows of Q or K
  static constexpr int V_CHUNKS = F8V ? D / 128 : CHUNKS;  // 128-byte boxes per V row
  static constexpr int V_ELEMS = F8V ? 128 : 64;
  static constexpr int V_BYTES = V_CHUNKS * 128 * 128;     // 128 rows of V
  static constexpr int NK = (D == 64 || F8) ? 2 : 1;       // K ring stages
  static constexpr int NV = (D == 64 || F8V) ? 2 : 1;      // V ring stages
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + QK_BYTES;
  static constexpr int OFF_V = OFF_K + NK * QK_BYTES;
  static constexpr int OFF_BAR = OFF_V + NV * V_BYTES;
  static constexpr int NBAR = 1 + 2 * NK + 2 * NV + 1 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int TOTAL = OFF_MISC + 16;
  static constexpr int ALLOC = TOTAL + 1024;
  static_assert(ALLOC <= (228 * 1024 - 2 * 1024) / 2, "two CTAs per SM must fit in shared memory");
};

template <int D, bool F8 = false, bool F8V = false>
__global__ void __launch_bounds__(NTHREADS, 2)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const Params p) {
  static_assert(!F8V || (F8 && D == 128), "e4m3 P*V comes with e4m3 Q*K^T at d = 128");
  using L = Smem2<D, F8, F8V>;
  constexpr int NK = L::NK, NV = L::NV;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  // qk_done[j % NK] completes when Q*K_j^T is done: S_j is in TMEM for the
  // softmax and K stage j % NK is free for the loader.  Each waits for a phase
  // before the barrier can complete the next one for that stage (block j+NK
  // needs K_{j+NK}, loaded after the loader's wait, and its Q*K^T is issued
  // after P_{j+NK-1}, produced after the softmax has read S_j).
  uint64_t* qk_done = k_full + NK;
  uint64_t* v_full = qk_done + NK;
  uint64_t* v_empty = v_full + NV;
  uint64_t* p_full = v_empty + NV;
  uint64_t* o_final = p_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  const int qblk = blockIdx.x;
  WaitCtx wc;
  wc.abort_flag = abort_flag;
  wc.timeout_ns = p.ctl.timeout_ns;
  wc.err_word = p.ctl.err_word;

  int q_tile, q_row0, q_valid, sub = 0;
  if (p.mode == FWD_STA) {
    q_tile = qblk / p.q_blocks_per_tile;
    sub = qblk - q_tile * p.q_blocks_per_tile;
    q_row0 = q_tile * p.g.s + sub * BM;
    q_valid = min(BM, p.g.s - sub * BM);
  } else {
    q_tile = 0;
    q_row0 = qblk * BM;
    q_valid = min(BM, p.g.N - q_row0);
  }
  const Stream st = fwd::make_stream(p, q_tile);
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
    mbar_init(p_full, 4);  // one arrival per softmax warp
    mbar_init(o_final, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == WARP_MMA) {
    tmem_alloc(tmem_slot, TMEM_COLS);
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

  constexpr uint32_t BOX_BYTES = 128 * 128;  // one 128-row x 128-byte box
  const uint32_t sub_bytes = (uint32_t)p.G * 128;
  const int subs = BN / p.G;

  if (warp >= 4) {
  reg_dealloc<REGS_OTHER>();
  if (warp == WARP_QK_LOAD) {
    if (lane == 0) {
      int issued_k = 0;
      if (!dcheck(fwd::query_block_ok(p, q_row0, q_valid), p.ctl.err_word)) *abort_flag = 1;
      if (!(p.ctl.debug_flags & 1) && !*abort_flag) {
        mbar_arrive_expect_tx(q_full, L::QK_BYTES);
        if (p.raster) {
          const DevGeom& g = p.g;
          const int at = q_tile / (g.Nh * g.Nw), ah = (q_tile / g.Nw) % g.Nh, aw = q_tile % g.Nw;
          const int t0 = at * g.tt + sub * BM / (g.th * g.tw);
          for (int c = 0; c < L::QK_CHUNKS; ++c)
            fwd::tma_load_5d(smem + L::OFF_Q + c * BOX_BYTES, &tm_q, q_full, c * L::QK_ELEMS, aw * g.tw, ah * g.th,
                             t0, bh);
        } else {
          for (int c = 0; c < L::QK_CHUNKS; ++c)
            tma_load_3d(smem + L::OFF_Q + c * BOX_BYTES, &tm_q, q_full, c * L::QK_ELEMS, q_row0, bh);
        }
      }
      for (int j = 0; j < nblk; ++j) {
        const int s = j % NK, r = j / NK;
        if (!mbar_wait(&qk_done[s], (r & 1) ^ 1, wc)) break;
        if (!dcheck(fwd::key_block_ok(p, st, j, L_total), p.ctl.err_word)) {
          *abort_flag = 1;
          break;
        }
        mbar_arrive_expect_tx(&k_full[s], L::QK_BYTES);
        uint8_t* dst = smem + L::OFF_K + s * L::QK_BYTES;
        for (int u = 0; u < subs; ++u) {
          const int v = j * BN + u * p.G;
          if (p.raster) {
            int x, y, t;
            fwd::stream_box(p, st, v, L_total, &x, &y, &t);
            for (int c = 0; c < L::QK_CHUNKS; ++c)
              fwd::tma_load_5d(dst + c * BOX_BYTES + u * sub_bytes, &tm_k, &k_full[s], c * L::QK_ELEMS, x, y, t, bh);
          } else {
            const int row = v < L_total ? fwd::stream_row(p, st, v) : p.Nk;  // past the end: zero fill
            for (int c = 0; c < L::QK_CHUNKS; ++c)
              tma_load_3d(dst + c * BOX_BYTES + u * sub_bytes, &tm_k, &k_full[s], c * L::QK_ELEMS, row, bh);
          }
        }
        ++issued_k;
      }
      // every issued load has landed before the CTA can exit (a no-op unless aborted)
      for (int j = issued_k - NK < 0 ? 0 : issued_k - NK; j < issued_k; ++j)
        mbar_wait_drain(&k_full[j % NK], (j / NK) & 1, wc);
    }
  } else if (warp == WARP_V_LOAD) {
    if (lane == 0) {
      int issued_v = 0;
      for (int j = 0; j < nblk; ++j) {
        const int s = j % NV, r = j / NV;
        if (!mbar_wait(&v_empty[s], (r & 1) ^ 1, wc)) break;
        if (!dcheck(fwd::key_block_ok(p, st, j, L_total), p.ctl.err_word)) {
          *abort_flag = 1;
          break;
        }
        mbar_arrive_expect_tx(&v_full[s], L::V_BYTES);
        uint8_t* dst = smem + L::OFF_V + s * L::V_BYTES;
        for (int u = 0; u < subs; ++u) {
          const int v = j * BN + u * p.G;
          if (p.raster) {
            int x, y, t;
            fwd::stream_box(p, st, v, L_total, &x, &y, &t);
            for (int c = 0; c < L::V_CHUNKS; ++c)
              fwd::tma_load_5d(dst + c * BOX_BYTES + u * sub_bytes, &tm_v, &v_full[s], c * L::V_ELEMS, x, y, t, bh);
          } else {
            const int row = v < L_total ? fwd::stream_row(p, st, v) : p.Nk;
            for (int c = 0; c < L::V_CHUNKS; ++c)
              tma_load_3d(dst + c * BOX_BYTES + u * sub_bytes, &tm_v, &v_full[s], c * L::V_ELEMS, row, bh);
          }
        }
        ++issued_v;
      }
      for (int j = issued_v - NV < 0 ? 0 : issued_v - NV; j < issued_v; ++j)
        mbar_wait_drain(&v_full[j % NV], (j / NV) & 1, wc);
    }
  } else if (warp == WARP_MMA) {
    if (lane == 0) {
      constexpr uint32_t IDESC_QK = idesc_bf16_f32(BM, BN, 0, 0);
      constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, D, 0, 1);
      const uint32_t q_base = smem_u32(smem + L::OFF_Q);
      const uint32_t k_base = smem_u32(smem + L::OFF_K);
      const uint32_t v_base = smem_u32(smem + L::OFF_V);
      const uint32_t s_tmem = tmem + S_COL, o_tmem = tmem + O_COL;
      bool ok = mbar_wait(q_full, 0, wc);
      auto issue_qk = [&](int j) -> bool {
        const int s = j % NK;
        if (!mbar_wait(&k_full[s], (j / NK) & 1, wc)) return false;
        tc_fence_after();
        const uint32_t kb = k_base + s * L::QK_BYTES;
        // four 32-byte K-steps per 128-byte box: 16 bf16 or 32 e4m3 elements each
#pragma unroll
        for (int kk = 0; kk < L::QK_CHUNKS * 4; ++kk) {
          const uint32_t off = (kk >> 2) * BOX_BYTES + (kk & 3) * 32;
          if constexpr (F8)
            fwd::mma_ss_e4m3(s_tmem, smem_desc_sw128(q_base + off, 16, 1024), smem_desc_sw128(kb + off, 16, 1024),
                             fwd::idesc_e4m3_f32(BM, BN), kk > 0);
          else
            mma_ss(s_tmem, smem_desc_sw128(q_base + off, 16, 1024), smem_desc_sw128(kb + off, 16, 1024), IDESC_QK,
                   kk > 0);
        }
        tc_commit(&qk_done[s]);
        return true;
      };
      if (ok && nblk > 0) ok = issue_qk(0);
      for (int j = 0; ok && j < nblk; ++j) {
        if (!mbar_wait(p_full, j & 1, wc)) break;
        const int s = j % NV;
        if (!mbar_wait(&v_full[s], (j / NV) & 1, wc)) break;
        tc_fence_after();
        const uint32_t vb = v_base + s * L::V_BYTES;
        if constexpr (F8V) {
          // e4m3: four K = 32 steps; A = P packed four to a TMEM column (8 columns
          // per step); B = V block (keys x d, one 128-byte row per key), MN-major,
          // SBO = next 8 keys
#pragma unroll
          for (int kk = 0; kk < BN / 32; ++kk)
            fwd::mma_ts_e4m3(o_tmem, s_tmem + kk * 8, smem_desc_sw128(vb + kk * 4096, BOX_BYTES, 1024),
                             fwd::idesc_e4m3_f32_bmn(BM, D), (j > 0 || kk > 0) ? 1u : 0u);
        } else {
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            // B = V block (keys x d), MN-major: LBO = next 64-column box, SBO = next 8 keys
            mma_ts(o_tmem, s_tmem + kk * 8, smem_desc_sw128(vb + kk * 2048, BOX_BYTES, 1024), IDESC_PV,
                   (j > 0 || kk > 0) ? 1u : 0u);
          }
        }
        tc_commit(&v_empty[s]);
        if (j + 1 < nblk) ok = issue_qk(j + 1);
      }
      tc_commit(o_final);
      // every MMA this thread issued must be finished before TMEM is freed
      mbar_wait_drain(o_final, 0, wc);
    }
  }
  } else {
    reg_alloc<REGS_SOFTMAX>();
    // ---------------- softmax: one row per thread ----------------
    const int quad = warp;
    const int row = quad * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    const uint32_t tS = tmem + lane_addr + S_COL;
    const uint32_t tO = tmem + lane_addr + O_COL;
    float c2 = p.scale_log2;
    if constexpr (F8) {  // S = bytes(Q) bytes(K)^T * (absmax_Q / 448) * (absmax_K / 448)
      const float aq = __int_as_float(p.qk_amax[2 * bh]), ak = __int_as_float(p.qk_amax[2 * bh + 1]);
      c2 *= (aq > 0.f ? aq / 448.f : 1.f) * (ak > 0.f ? ak / 448.f : 1.f);
    }
    // e4m3 P: the running max moves when a row's max grows by more than 2^2,
    // so P <= 2^2 and P * 2^6 <= 2^8 < 448 (the largest e4m3); the factor 2^6
    // (folded into the exponent) keeps small probabilities out of e4m3's
    // subnormal range and cancels against the row sum, which is accumulated in
    // the same units.
    constexpr float THRESH = F8V ? 2.0f : RESCALE_LOG2_THRESHOLD;
    constexpr float PSHIFT = F8V ? 6.0f : 0.0f;
    float m_ref = -INFINITY, l_sum = 0.f;
    bool ok = true;
    for (int j = 0; j < nblk; ++j) {
      ok = mbar_wait(&qk_done[j % NK], (j / NK) & 1, wc);
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
      if (j == 0) {
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
          if ((POLY_MASK >> q4) & 1) {  // FMA-pipe exponentials for this chunk
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
        // O is quiescent: the commit that signalled this S also covers the
        // previous P*V into O, and the next one waits for p_full.
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
      if (lane == 0) mbar_arrive(p_full);
    }
    // ---------------- epilogue ----------------
    if (ok && !*abort_flag) ok = mbar_wait(o_final, 0, wc);
    ok = __all_sync(0xffffffffu, ok);
    tc_fence_after();
    if (ok && !*abort_flag) {
      float inv_l = 1.f / l_sum;
      if constexpr (F8V) {  // O = P V with V = bytes(V) * absmax_V / 448
        const float av = __int_as_float(p.v_amax[bh]);
        inv_l *= av > 0.f ? av / 448.f : 1.f;
      }
      bool row_ok = row < q_valid;
      size_t grow = (size_t)bh * p.g.N + (size_t)(q_row0 + row);
      if (p.raster) {  // tile-major row -> raster token
        const DevGeom& g = p.g;
        const int at = q_tile / (g.Nh * g.Nw), ah = (q_tile / g.Nw) % g.Nh, aw = q_tile % g.Nw;
        const int lr = sub * BM + row;
        const int lt = lr / (g.th * g.tw), lh = (lr / g.tw) % g.th, lw = lr % g.tw;
        grow = (size_t)bh * g.N + ((size_t)(at * g.tt + lt) * g.H + (ah * g.th + lh)) * g.W + (aw * g.tw + lw);
      }
      if (row_ok && !dcheck(fwd::out_row_ok(p, bh, grow), p.ctl.err_word)) row_ok = false;
      // hierarchical merge: one softmax over the fine keys (O_f, LSE_f given)
      // and this kernel's coarse keys, in log2 units
      float wf = 0.f, wk = 1.f, lse2_out = m_ref - PSHIFT + __log2f(l_sum);
      if (p.merge_o && row_ok) {
        const float lf2 = p.merge_lse[grow] * 1.4426950408889634f;
        const float mm = fmaxf(lf2, lse2_out);
        wf = ex2(lf2 - mm);
        wk = ex2(lse2_out - mm);
        const float inv = 1.f / (wf + wk);
        lse2_out = mm + __log2f(wf + wk);
        wf *= inv;
        wk *= inv;
      }
      float gh = 0.f;
      if (p.blend_out) gh = p.gvec[bh % p.g.heads];
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t x0[32];
        tmem_ld32(tO + c0, x0);
        tmem_wait_ld();
        float* o = reinterpret_cast<float*>(x0);
#pragma unroll
        for (int c = 0; c < 32; ++c) o[c] = __uint_as_float(x0[c]) * inv_l;
        if (row_ok && p.merge_o) {
          const uint4* src = reinterpret_cast<const uint4*>(p.merge_o + grow * D + c0);
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4) {
            const uint4 of = src[v4];
            const uint32_t w4[4] = {of.x, of.y, of.z, of.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              o[8 * v4 + 2 * e] = wf * bf16lo(w4[e]) + wk * o[8 * v4 + 2 * e];
              o[8 * v4 + 2 * e + 1] = wf * bf16hi(w4[e]) + wk * o[8 * v4 + 2 * e + 1];
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
      if (row_ok && p.lse) p.lse[grow] = lse2_out * 0.69314718055994531f;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace fwd2

// Launches the two-CTA kernel on parameters prepared by the common forward
// launcher (tensor maps encoded, Params filled in).
template <int D, bool F8, bool F8V>
cudaError_t launch_fwd2(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const fwd::Params& p,
                        dim3 grid, cudaStream_t st) {
  using L = fwd2::Smem2<D, F8, F8V>;
  auto kernel = fwd2::attn_fwd_kernel<D, F8, F8V>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e != cudaSuccess) return e;
  kernel<<<grid, fwd2::NTHREADS, L::ALLOC, st>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

template cudaError_t launch_fwd2<128, false, false>(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                                                    const fwd::Params&, dim3, cudaStream_t);
template cudaError_t launch_fwd2<64, false, false>(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                                                   const fwd::Params&, dim3, cudaStream_t);
template cudaError_t launch_fwd2<128, true, false>(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                                                   const fwd::Params&, dim3, cudaStream_t);
template cudaError_t launch_fwd2<128, true, true>(const CUtensorMap&, const CUtensorMap&, const CUtensorMap&,
                                                  const fwd::Params&, dim3, cudaStream_t);

// Resident CTAs per SM of the two-CTA kernel (occupancy check for tests).
template <int D, bool F8, bool F8V = false>
static int ctas_per_sm() {
  using L = fwd2::Smem2<D, F8, F8V>;
  auto kernel = fwd2::attn_fwd_kernel<D, F8, F8V>;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC) != cudaSuccess ||
      cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess)
    return -1;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, fwd2::NTHREADS, L::ALLOC) != cudaSuccess) return -1;
  return n;
}

int fwd2_ctas_per_sm(int d, bool f8) {
  if (f8) return d == 128 ? std::min(ctas_per_sm<128, true>(), ctas_per_sm<128, true, true>()) : -1;
  if (d == 64) return ctas_per_sm<64, false>();
  if (d == 128) return ctas_per_sm<128, false>();
  return -1;
}

}  // namespace vattn

// Attention backward on tcgen05 tensor cores.
//
// Gradients of O = g*O_l + (1-g)*O_g ("UltraGen ..." §4.1) with the softmax
// attention of each branch restated per branch b with weight gamma_b
// (gamma_l = g, gamma_g = 1 - g; gamma = 1 for the sliding-tile backward):
//   D_b   = rowsum(dO * O_b)
//   P_b   = exp(S_b - LSE_b),  dP_b = dO V_b^T
//   dS_b  = gamma_b * P_b * (dP_b - D_b)
//   dV_b  = gamma_b * P_b^T dO,  dK_b = scale * dS_b^T Q,  dQ = scale * sum_b dS_b K_b
// and the pooled branch's dK_p/dV_p flow back to every token of their pool
// block divided by its size.
//
// Kernels:
//   bwd_preprocess_kernel  D_l, D_g (and dg) from dO, O_l, O_g        HBM-bound
//   dkdv_kernel<D, PAIR>   one CTA per 128 keys; streams 64-query blocks:
//                          GLOBAL  -> all queries vs pooled keys, fp32 dK_p/dV_p
//                          LOCAL   -> the query tiles whose window holds the key
//                                     tile ("inverse window"), pool-backward
//                                     fused into the epilogue; PAIR: key blocks
//                                     of two w-adjacent 192-row tiles shared
//                          HIER    -> coarse keys, fp32 dK_h/dV_h
//   dq_kernel<D, PAIR>     one CTA per 128 queries; streams 96-key blocks:
//                          GLOBAL  -> all pooled keys, fp32 partial dQ out
//                          LOCAL   -> the kept window, adding the global part;
//                                     PAIR: query blocks shared as in the forward
//                          HIER    -> the coarse window, fp32 partial dQ out
// TMEM holds S/dP double-buffered per softmax group plus the accumulators;
// P and dS are written back as bf16 over their own S/dP columns and read by
// the next MMAs as the A operand.  No atomics: dQ, dK and dV are
// deterministic.
#include "bwd_common.cuh"

namespace vattn {

namespace bwd {

constexpr int NTHREADS = 352;
constexpr int WARP_LOAD_A = 8;
constexpr int WARP_LOAD_B = 9;
constexpr int WARP_MMA = 10;
// ---------------------------------------------------------------------------
// preprocess: D_l, D_g, dg
// ---------------------------------------------------------------------------
// grid (blocks_per_bh, B*heads); every group of vpr = d/8 lanes handles one row.
// It writes the negated row terms -D_b and -L_b with
// L_b = LSE_b*log2(e) - log2(gamma_b), so that the kernels form
// gamma_b*P_b = exp2(S*scale*log2(e) - L_b) with one FMA and one ex2 and
// dS_b = gamma_b*P_b*(dP_b - D_b) with one add and one multiply (gamma_b = 0
// gives L_b = +inf and gamma_b*P_b = 0).
struct PreArgs {
  const uint4* dout;
  const uint4* o_l;
  const uint4* o_g;       // NULL: single branch
  const float* lse_l;
  const float* lse_g;
  float* ndelta_l;
  float* ndelta_g;
  float* nlse2_l;
  float* nlse2_g;
  float* dg;              // NULL: skip
  const float* gvec;      // NULL: gamma_l = 1
  int vpr, N, heads;
};

__global__ void __launch_bounds__(256, 8) bwd_preprocess_kernel(const PreArgs a) {
  const int bh = blockIdx.y;
  const int h = bh % a.heads;
  const int groups = blockDim.x / a.vpr;
  const int grp = threadIdx.x / a.vpr, lane_in = threadIdx.x % a.vpr;
  const float gl = a.gvec ? a.gvec[h] : 1.f, gg = 1.f - gl;
  const float off_l = __log2f(gl), off_g = __log2f(gg);
  float dg_acc = 0.f;
  // the loop bound is uniform across the block, so every lane reaches the
  // shuffles; rows past the end contribute zero
  for (int rb = blockIdx.x * groups; rb < a.N; rb += gridDim.x * groups) {
    const int r = rb + grp;
    const bool in = r < a.N;
    float sl = 0.f, sg = 0.f;
    // the row's LSE values are fetched with its vectors, so the loop waits
    // once per row on memory, not twice
    float lse_l = 0.f, lse_g = 0.f;
    if (in && lane_in == 0) {
      const size_t i = (size_t)bh * a.N + r;
      lse_l = __ldg(a.lse_l + i);
      if (a.o_g) lse_g = __ldg(a.lse_g + i);
    }
    if (in) {
      const size_t base = ((size_t)bh * a.N + r) * a.vpr + lane_in;
      const uint4 x = __ldg(a.dout + base);
      const uint4 y = __ldg(a.o_l + base);
      const uint32_t xv[4] = {x.x, x.y, x.z, x.w}, yv[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) sl += bf16lo(xv[e]) * bf16lo(yv[e]) + bf16hi(xv[e]) * bf16hi(yv[e]);
      if (a.o_g) {
        const uint4 z = __ldg(a.o_g + base);
        const uint32_t zv[4] = {z.x, z.y, z.z, z.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) sg += bf16lo(xv[e]) * bf16lo(zv[e]) + bf16hi(xv[e]) * bf16hi(zv[e]);
      }
    }
    for (int o = a.vpr / 2; o > 0; o >>= 1) {
      sl += __shfl_xor_sync(0xffffffffu, sl, o);
      sg += __shfl_xor_sync(0xffffffffu, sg, o);
    }
    if (in && lane_in == 0) {
      const size_t i = (size_t)bh * a.N + r;
      a.ndelta_l[i] = -sl;
      a.nlse2_l[i] = off_l - lse_l * LOG2E;
      if (a.o_g) {
        a.ndelta_g[i] = -sg;
        a.nlse2_g[i] = off_g - lse_g * LOG2E;
      }
      dg_acc += sl - sg;
    }
  }
  if (a.dg) {
    __shared__ float red[32];
    for (int o = 16; o > 0; o >>= 1) dg_acc += __shfl_xor_sync(0xffffffffu, dg_acc, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = dg_acc;
    __syncthreads();
    if (threadIdx.x == 0) {
      float t = 0.f;
      for (int i = 0; i < (int)(blockDim.x >> 5); ++i) t += red[i];
      atomicAdd(&a.dg[h], t);
    }
  }
}

// ---------------------------------------------------------------------------
// dK / dV
// ---------------------------------------------------------------------------
template <int D>
struct DkdvSmem {
  static constexpr int CHUNKS = D / 64;
  static constexpr int KV_BYTES = CHUNKS * 128 * 128;  // 128 key rows
  static constexpr int QB_BYTES = CHUNKS * 64 * 128;   // 64 query rows
  static constexpr int NQ = 3;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = KV_BYTES;
  static constexpr int OFF_Q = 2 * KV_BYTES;
  static constexpr int OFF_DO = OFF_Q + NQ * QB_BYTES;
  static constexpr int OFF_LSE = OFF_DO + NQ * QB_BYTES;
  static constexpr int OFF_DEL = OFF_LSE + NQ * 256;
  static constexpr int OFF_BAR = OFF_DEL + NQ * 256;
  static constexpr int NBAR = 1 + 2 * NQ + 2 + 2 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int TOTAL = OFF_MISC + 16;
  static constexpr int ALLOC = TOTAL + 1024;
};

template <int D, bool PAIR = false>
__global__ void __launch_bounds__(NTHREADS, 1)
    dkdv_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                const DkdvParams p) {
  using L = DkdvSmem<D>;
  constexpr int NQ = L::NQ;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* kv_full = bars;
  // One full / empty pair per query stage for Q, dO and the L / D rows: the two
  // loader warps each arrive (with their byte counts) on the same full
  // barrier, and one commit releases the whole stage.  Every barrier wait or
  // commit costs the MMA thread about as long as an MMA, and the tensor pipe
  // holds little more than one MMA in flight, so fewer of them per block keep
  // the pipe busier.
  uint64_t* qd_full = bars + 1;
  uint64_t* qd_empty = qd_full + NQ;
  uint64_t* sdp_full = qd_empty + NQ;
  uint64_t* p_full = sdp_full + 2;
  uint64_t* acc_done = p_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);
  float* lse_s = reinterpret_cast<float*>(smem + L::OFF_LSE);
  float* del_s = reinterpret_cast<float*>(smem + L::OFF_DEL);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  const DevGeom& g = p.g;
  WaitCtx wc;
  wc.abort_flag = abort_flag;
  wc.timeout_ns = p.ctl.timeout_ns;
  wc.err_word = p.ctl.err_word;

  int key_row0, key_valid;
  RowStream qs;
  // PAIR, straddling key block (keys [0, 64) of tile a, [64, 128) of tile
  // a + 1): the query stream is the union of the two inverse windows, which
  // along w are contiguous and nested in order; the first tile's key rows
  // (quads 0, 1) skip run offsets >= xa, the second's (quads 2, 3) offsets < xb
  int xa = 0, xb = 0;
  bool kmask = false;
  if (PAIR && p.mode == DKDV_LOCAL) {
    const QueryBlock kb = paired_query_block(g, p.pair, blockIdx.x);  // key blocks, same layout
    key_row0 = kb.row0;
    key_valid = kb.valid;
    qs = inverse_stream(g, p.gk, 1, 1, 1, kb.tile);
    if (kb.straddle) {
      const RowStream q2 = inverse_stream(g, p.gk, 1, 1, 1, kb.tile + 1);
      xa = qs.run_len;
      xb = (q2.w0 - qs.w0) * g.s;
      qs.run_len = xb + q2.run_len;
      kmask = xa < qs.run_len || xb > 0;
    }
  } else if (p.mode != DKDV_GLOBAL) {
    const int kt = blockIdx.x / p.kv_blocks_per_tile;
    const int sb = blockIdx.x - kt * p.kv_blocks_per_tile;
    key_row0 = kt * g.s + sb * 128;
    key_valid = min(128, g.s - sb * 128);
    qs = inverse_stream(g, p.gk, p.cft, p.cfh, p.cfw, kt);
  } else {
    key_row0 = blockIdx.x * 128;
    key_valid = min(128, p.Nk - key_row0);
    qs = flat_stream(g.N);
  }
  const int Lq = qs.length();
  const int nblk = (Lq + 63) / 64;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int i = 0; i < NQ; ++i) {
      mbar_init(&qd_full[i], 2);  // one arrival per loader warp
      mbar_init(&qd_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sdp_full[i], 1);
      mbar_init(&p_full[i], 4);  // one arrival per softmax warp
    }
    mbar_init(acc_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == WARP_MMA) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  constexpr uint32_t KBOX = 128 * 128;  // 128 rows x 128 bytes
  constexpr uint32_t QBOX = 64 * 128;   // 64 rows x 128 bytes
  const int subs = 64 / p.Gq;

  if (warp == WARP_LOAD_A || warp == WARP_LOAD_B) {
    if (lane == 0) {
      const bool is_a = warp == WARP_LOAD_A;  // A: K, V tiles, Q and LSE; B: dO and D
      if (is_a && dcheck(key_row0 >= 0 && key_row0 < p.Nk, p.ctl.err_word)) {
        mbar_arrive_expect_tx(kv_full, 2 * L::KV_BYTES);
        for (int c = 0; c < L::CHUNKS; ++c) {
          tma_load_3d(smem + L::OFF_K + c * KBOX, &tm_k, kv_full, c * 64, key_row0, bh);
          tma_load_3d(smem + L::OFF_V + c * KBOX, &tm_v, kv_full, c * 64, key_row0, bh);
        }
      }
      uint64_t* full = qd_full;
      uint64_t* empty = qd_empty;
      const CUtensorMap* tm = is_a ? &tm_q : &tm_do;
      const float* vec = is_a ? p.nlse2 : p.ndelta;
      float* vec_s = is_a ? lse_s : del_s;
      const uint32_t off_x = is_a ? L::OFF_Q : L::OFF_DO;
      int issued = 0;
      if (is_a && !dcheck(key_row0 >= 0 && key_valid > 0 && key_row0 + key_valid <= p.Nk, p.ctl.err_word))
        *abort_flag = 1;
      for (int i = 0; i < nblk && !*abort_flag; ++i) {
        const int s = i % NQ, r = i / NQ;
        if (!mbar_wait(&empty[s], (r & 1) ^ 1, wc)) break;
        if constexpr (kDebugChecks) {
          bool good = true;
          for (int u = 0; u < subs; ++u) good = good && stream_box_ok(qs, g, i * 64 + u * p.Gq, p.Gq, Lq, g.N);
          if (!dcheck(good, p.ctl.err_word)) {
            *abort_flag = 1;
            break;
          }
        }
        // LSE / D rows: whole 16-byte groups by bulk copy when the source is
        // 16-byte aligned; a ragged tail (end of a flat query stream) or an
        // unaligned source (a pooled grid used as the token sequence, N_p not
        // a multiple of 4) by plain loads, written before the arrival that
        // publishes the stage.
        uint32_t tx = L::QB_BYTES;
        int nbulk[4] = {0, 0, 0, 0};  // subs <= 4 (Gq >= 16)
        for (int u = 0; u < subs; ++u) {
          const int v = i * 64 + u * p.Gq;
          if (v >= Lq) break;
          const int n = min(p.Gq, Lq - v);
          const size_t gi = (size_t)bh * g.N + qs.row(g, v);
          const int nb = (gi % 4 == 0) ? (n & ~3) : 0;
          nbulk[u] = nb;
          tx += nb * 4;
          for (int t = nb; t < n; ++t) vec_s[s * 64 + u * p.Gq + t] = vec[gi + t];
        }
        mbar_arrive_expect_tx(&full[s], tx);
        for (int u = 0; u < subs; ++u) {
          const int v = i * 64 + u * p.Gq;
          const bool ok = v < Lq;
          const int row = ok ? qs.row(g, v) : g.N;
          for (int c = 0; c < L::CHUNKS; ++c)
            tma_load_3d(smem + off_x + s * L::QB_BYTES + c * QBOX + u * p.Gq * 128, tm, &full[s], c * 64, row, bh);
          if (ok && nbulk[u] > 0)
            bulk_load(vec_s + s * 64 + u * p.Gq, vec + (size_t)bh * g.N + row, nbulk[u] * 4, &full[s]);
        }
        ++issued;
      }
      for (int i = issued - NQ < 0 ? 0 : issued - NQ; i < issued; ++i) mbar_wait_drain(&full[i % NQ], (i / NQ) & 1, wc);
      if (is_a) mbar_wait_drain(kv_full, 0, wc);
    }
  } else if (warp == WARP_MMA) {
    if (lane == 0) {
      constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 64, 0, 0);
      constexpr uint32_t IDESC_ACC = idesc_bf16_f32(128, D, 0, 1);
      const uint32_t k_base = smem_u32(smem + L::OFF_K), v_base = smem_u32(smem + L::OFF_V);
      const uint32_t q_base = smem_u32(smem + L::OFF_Q), do_base = smem_u32(smem + L::OFF_DO);
      bool ok = mbar_wait(kv_full, 0, wc);
      auto issue_sdp = [&](int i) -> bool {
        const int s = i % NQ, w = i & 1;
        if (!mbar_wait(&qd_full[s], (i / NQ) & 1, wc)) return false;
        tc_fence_after();
        const uint32_t qb = q_base + s * L::QB_BYTES, db = do_base + s * L::QB_BYTES;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t ko = (kk >> 2) * KBOX + (kk & 3) * 32, qo = (kk >> 2) * QBOX + (kk & 3) * 32;
          mma_ss(tmem + w * 64, smem_desc_sw128(k_base + ko, 16, 1024), smem_desc_sw128(qb + qo, 16, 1024), IDESC_S,
                 kk > 0);
          mma_ss(tmem + 128 + w * 64, smem_desc_sw128(v_base + ko, 16, 1024), smem_desc_sw128(db + qo, 16, 1024),
                 IDESC_S, kk > 0);
        }
        tc_commit(&sdp_full[w]);
        return true;
      };
      if (ok) ok = issue_sdp(0);
      if (ok && nblk > 1) ok = issue_sdp(1);
      for (int i = 0; ok && i < nblk; ++i) {
        const int w = i & 1, s = i % NQ;
        if (!mbar_wait(&p_full[w], (i >> 1) & 1, wc)) break;
        tc_fence_after();
        const uint32_t qb = q_base + s * L::QB_BYTES, db = do_base + s * L::QB_BYTES;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          // dV += P^T dO ; dK += dS^T Q   (B operands MN-major: LBO = next 64-column box)
          mma_ts(tmem + 256, tmem + w * 64 + kk * 8, smem_desc_sw128(db + kk * 2048, QBOX, 1024), IDESC_ACC,
                 (i > 0 || kk > 0) ? 1u : 0u);
          mma_ts(tmem + 384, tmem + 128 + w * 64 + kk * 8, smem_desc_sw128(qb + kk * 2048, QBOX, 1024), IDESC_ACC,
                 (i > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(&qd_empty[s]);
        if (i + 2 < nblk) ok = issue_sdp(i + 2);
      }
      tc_commit(acc_done);
      mbar_wait_drain(acc_done, 0, wc);
    }
  } else {
    // ---------------- softmax groups: row = key ----------------
    const int w = warp >> 2, quad = warp & 3, row = quad * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    const uint32_t tS = tmem + lane_addr + (uint32_t)(w * 64);
    const uint32_t tP = tmem + lane_addr + 128u + (uint32_t)(w * 64);
    bool ok = true;
    int o_blk = (PAIR && kmask) ? (w * 64) % qs.run_len : 0;  // run offset of this group's block
    for (int i = w; i < nblk; i += 2) {
      const int it = i >> 1, s = i % NQ;
      ok = mbar_wait(&sdp_full[w], it & 1, wc);
      ok = ok && mbar_wait(&qd_full[s], (i / NQ) & 1, wc);   // L and D rows in shared memory
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const float2 c2x2 = make_float2(p.c2, p.c2);
      const float4* ls4 = reinterpret_cast<const float4*>(lse_s + s * 64);
      const float4* ds4 = reinterpret_cast<const float4*>(del_s + s * 64);
      int valid = Lq - i * 64;
      if (PAIR && kmask) {
        // a 64-query block lies in one query tile (s is a multiple of 64): the
        // whole block is outside this warp's key rows' window or inside it
        if ((quad >> 1) ? o_blk < xb : o_blk >= xa) valid = 0;
        o_blk += 128;  // this group's next block
        while (o_blk >= qs.run_len) o_blk -= qs.run_len;
      }
      const bool full_blk = valid >= 64;   // uniform: the last block, or a masked one
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        if (PAIR && valid <= 0) {  // whole block outside this warp's window: P = dS = 0, no exponentials
          const uint32_t z[16] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
          tmem_st16(tS + hh * 16, z);
          tmem_st16(tP + hh * 16, z);
          continue;
        }
        // one 32-column half at a time keeps S, dP and the packed outputs in registers
        uint32_t sv[32], dv[32];
        tmem_ld32(tS + hh * 32, sv);
        tmem_ld32(tP + hh * 32, dv);
        tmem_wait_ld();
        uint32_t pk[16], dk[16];
#pragma unroll
        for (int c4 = 0; c4 < 8; ++c4) {
          const float4 l4 = ls4[hh * 8 + c4], d4 = ds4[hh * 8 + c4];  // -L, -D of four query columns
#pragma unroll
          for (int e2 = 0; e2 < 2; ++e2) {
            const int c = c4 * 4 + e2 * 2;
            const float2 nl = e2 ? make_float2(l4.z, l4.w) : make_float2(l4.x, l4.y);
            const float2 nd = e2 ? make_float2(d4.z, d4.w) : make_float2(d4.x, d4.y);
            const float2 x = ffma2(make_float2(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1])), c2x2, nl);
            float2 pp = make_float2(ex2(x.x), ex2(x.y));
            float2 dd = fmul2(pp, fadd2(make_float2(__uint_as_float(dv[c]), __uint_as_float(dv[c + 1])), nd));
            if (!full_blk) {
              const int cc = hh * 32 + c;
              if (cc >= valid) pp.x = dd.x = 0.f;
              if (cc + 1 >= valid) pp.y = dd.y = 0.f;
            }
            pk[c4 * 2 + e2] = pack_bf16(pp.x, pp.y);
            dk[c4 * 2 + e2] = pack_bf16(dd.x, dd.y);
          }
        }
        tmem_st16(tS + hh * 16, pk);
        tmem_st16(tP + hh * 16, dk);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[w]);
    }
    // ---------------- epilogue: group 0 writes dV, group 1 writes dK ----------------
    if (ok && !*abort_flag) ok = mbar_wait(acc_done, 0, wc);
    ok = __all_sync(0xffffffffu, ok);
    tc_fence_after();
    if (ok && !*abort_flag) {
      const bool row_ok = row < key_valid;
      const uint32_t tAcc = tmem + lane_addr + (w == 0 ? 256u : 384u);
      const float mul = (w == 0) ? 1.f : p.scale;
      const size_t tok = (size_t)key_row0 + row;
      if (p.mode != DKDV_LOCAL) {
        float* dst = (w == 0 ? p.dvp_out : p.dkp_out) + ((size_t)bh * p.Nk + tok) * D;
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t x[32];
          tmem_ld32(tAcc + c0, x);
          tmem_wait_ld();
          if (row_ok) {
#pragma unroll
            for (int v4 = 0; v4 < 8; ++v4)
              reinterpret_cast<float4*>(dst + c0)[v4] =
                  make_float4(__uint_as_float(x[4 * v4]) * mul, __uint_as_float(x[4 * v4 + 1]) * mul,
                              __uint_as_float(x[4 * v4 + 2]) * mul, __uint_as_float(x[4 * v4 + 3]) * mul);
          }
        }
      } else {
        const float* add = (w == 0) ? p.dvp_in : p.dkp_in;
        const float* add_row = nullptr;
        float inv_cnt = 0.f;
        if (add && row_ok) {
          const int prow = p.hier_add ? coarse_of_tiled(g, p.gadd, (int)tok) : pooled_of_tiled(g, (int)tok);
          if (dcheck(prow >= 0 && prow < g.Np, p.ctl.err_word)) add_row = add + ((size_t)bh * g.Np + prow) * D;
          inv_cnt = 1.f / (float)(g.pt * g.ph * g.pw);
        }
        __nv_bfloat16* dst = (w == 0 ? p.dv : p.dk) + ((size_t)bh * g.N + tok) * D;
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t x[32];
          tmem_ld32(tAcc + c0, x);
          tmem_wait_ld();
          if (row_ok) {
            float f[32];
#pragma unroll
            for (int c = 0; c < 32; ++c) f[c] = __uint_as_float(x[c]) * mul;
            if (add_row) {
#pragma unroll
              for (int v4 = 0; v4 < 8; ++v4) {
                const float4 a = __ldg(reinterpret_cast<const float4*>(add_row + c0) + v4);
                f[4 * v4] += a.x * inv_cnt;
                f[4 * v4 + 1] += a.y * inv_cnt;
                f[4 * v4 + 2] += a.z * inv_cnt;
                f[4 * v4 + 3] += a.w * inv_cnt;
              }
            }
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4)
              reinterpret_cast<uint4*>(dst + c0)[v4] =
                  make_uint4(pack_bf16(f[8 * v4], f[8 * v4 + 1]), pack_bf16(f[8 * v4 + 2], f[8 * v4 + 3]),
                             pack_bf16(f[8 * v4 + 4], f[8 * v4 + 5]), pack_bf16(f[8 * v4 + 6], f[8 * v4 + 7]));
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// dQ
// ---------------------------------------------------------------------------
// dQ key block: 96 keys.  TMEM holds S0 [0,96), S1 [96,192), dP0 [192,288),
// dP1 [288,384) and the dQ accumulator [384,384+D); a 96-wide block puts 50%
// more work into every S / dP instruction than a 64-wide one.
constexpr int DQ_BN = 96;
constexpr uint32_t DQ_S0 = 0, DQ_S1 = 96, DQ_P0 = 192, DQ_P1 = 288, DQ_ACC = 384;

template <int D>
struct DqSmem {
  static constexpr int CHUNKS = D / 64;
  static constexpr int QB_BYTES = CHUNKS * 128 * 128;    // 128 query rows
  static constexpr int KB_BYTES = CHUNKS * DQ_BN * 128;  // DQ_BN key rows
  static constexpr int NK = 3;
  static constexpr int NV = 3;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_DO = QB_BYTES;
  static constexpr int OFF_K = 2 * QB_BYTES;
  static constexpr int OFF_V = OFF_K + NK * KB_BYTES;
  static constexpr int OFF_BAR = OFF_V + NV * KB_BYTES;
  static_assert(NK == NV, "K and V stages share their barriers");
  static constexpr int NBAR = 1 + 2 * NK + 2 + 2 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int TOTAL = OFF_MISC + 16;
  static constexpr int ALLOC = TOTAL + 1024;
};

template <int D, bool PAIR = false>
__global__ void __launch_bounds__(NTHREADS, 1)
    dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
              const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
              const DqParams p) {
  using L = DqSmem<D>;
  constexpr int NK = L::NK, NV = L::NV;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* qdo_full = bars;
  // K and V of key block j share stage j % NK: one full barrier that both
  // loader warps arrive on, and one empty barrier committed after the dQ
  // product (the last reader of K) -- one wait and one commit per block
  // fewer for the MMA thread.
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = kv_full + NK;
  uint64_t* sdp_full = kv_empty + NK;
  uint64_t* p_full = sdp_full + 2;
  uint64_t* acc_done = p_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  const DevGeom& g = p.g;
  WaitCtx wc;
  wc.abort_flag = abort_flag;
  wc.timeout_ns = p.ctl.timeout_ns;
  wc.err_word = p.ctl.err_word;

  const bool glob = p.mode == DQ_GLOBAL;
  int q_row0, q_valid, q_tile = 0;
  bool straddle = false;
  if (glob) {
    q_row0 = blockIdx.x * 128;
    q_valid = min(128, g.N - q_row0);
  } else if (PAIR) {  // w-adjacent tiles share their query blocks (PairPlan)
    const QueryBlock qb = paired_query_block(g, p.pair, blockIdx.x);
    q_tile = qb.tile;
    q_row0 = qb.row0;
    q_valid = qb.valid;
    straddle = qb.straddle;
  } else {
    q_tile = blockIdx.x / p.q_blocks_per_tile;
    const int sub = blockIdx.x - q_tile * p.q_blocks_per_tile;
    q_row0 = q_tile * g.s + sub * 128;
    q_valid = min(128, g.s - sub * 128);
  }
  RowStream ks = glob ? flat_stream(g.Np) : window_stream(g, p.gk, p.cft, p.cfh, p.cfw, q_tile);
  if (PAIR && straddle && straddle_shift(g, p.gk.Nw, p.cfw, q_tile) != 0) {
    ks.rot = 1;
    ks.run_len += p.gk.s;
  }
  const int Lk = ks.length();
  const int nblk = (Lk + DQ_BN - 1) / DQ_BN;

  if (threadIdx.x == 0) {
    mbar_init(qdo_full, 1);
    for (int i = 0; i < NK; ++i) {
      mbar_init(&kv_full[i], 2);  // one arrival per loader warp
      mbar_init(&kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sdp_full[i], 1);
      mbar_init(&p_full[i], 4);  // one arrival per softmax warp
    }
    mbar_init(acc_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == WARP_MMA) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  constexpr uint32_t QBOX = 128 * 128;
  constexpr uint32_t KBOX = DQ_BN * 128;

  if (warp == WARP_LOAD_A || warp == WARP_LOAD_B) {
    if (lane == 0) {
      const bool is_k = warp == WARP_LOAD_A;
      if (is_k && !dcheck(q_row0 >= 0 && q_valid > 0 && q_row0 + q_valid <= g.N, p.ctl.err_word)) *abort_flag = 1;
      if (is_k && !*abort_flag) {
        mbar_arrive_expect_tx(qdo_full, 2 * L::QB_BYTES);
        for (int c = 0; c < L::CHUNKS; ++c) {
          tma_load_3d(smem + L::OFF_Q + c * QBOX, &tm_q, qdo_full, c * 64, q_row0, bh);
          tma_load_3d(smem + L::OFF_DO + c * QBOX, &tm_do, qdo_full, c * 64, q_row0, bh);
        }
      }
      const int NS = is_k ? NK : NV;
      uint64_t* full = kv_full;
      uint64_t* empty = kv_empty;
      const uint32_t off = is_k ? L::OFF_K : L::OFF_V;
      int issued = 0;
      for (int j = 0; j < nblk; ++j) {
        const int s = j % NS, r = j / NS;
        if (!mbar_wait(&empty[s], (r & 1) ^ 1, wc)) break;
        const int G = glob ? DQ_BN : p.G0;
        const CUtensorMap* tm = is_k ? &tm_k : &tm_v;
        const int oob = glob ? g.Np : p.gk.N;
        if constexpr (kDebugChecks) {
          bool good = true;
          for (int u = 0; u < DQ_BN / G; ++u) good = good && stream_box_ok(ks, p.gk, j * DQ_BN + u * G, G, Lk, oob);
          if (!dcheck(good, p.ctl.err_word)) {
            *abort_flag = 1;
            break;
          }
        }
        mbar_arrive_expect_tx(&full[s], L::KB_BYTES);
        for (int u = 0; u < DQ_BN / G; ++u) {
          const int v = j * DQ_BN + u * G;
          const int row = v < Lk ? ks.row(p.gk, v) : oob;
          for (int c = 0; c < L::CHUNKS; ++c)
            tma_load_3d(smem + off + s * L::KB_BYTES + c * KBOX + u * G * 128, tm, &full[s], c * 64, row, bh);
        }
        ++issued;
      }
      for (int j = issued - NS < 0 ? 0 : issued - NS; j < issued; ++j) mbar_wait_drain(&full[j % NS], (j / NS) & 1, wc);
      if (is_k) mbar_wait_drain(qdo_full, 0, wc);
    }
  } else if (warp == WARP_MMA) {
    if (lane == 0) {
      constexpr uint32_t IDESC_S = idesc_bf16_f32(128, DQ_BN, 0, 0);
      constexpr uint32_t IDESC_ACC = idesc_bf16_f32(128, D, 0, 1);
      const uint32_t q_base = smem_u32(smem + L::OFF_Q), do_base = smem_u32(smem + L::OFF_DO);
      const uint32_t k_base = smem_u32(smem + L::OFF_K), v_base = smem_u32(smem + L::OFF_V);
      bool ok = mbar_wait(qdo_full, 0, wc);
      auto issue_sdp = [&](int j) -> bool {
        const int w = j & 1, sk = j % NK, sv = sk;
        if (!mbar_wait(&kv_full[sk], (j / NK) & 1, wc)) return false;
        tc_fence_after();
        const uint32_t kb = k_base + sk * L::KB_BYTES, vb = v_base + sv * L::KB_BYTES;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t qo = (kk >> 2) * QBOX + (kk & 3) * 32, ko = (kk >> 2) * KBOX + (kk & 3) * 32;
          mma_ss(tmem + (w ? DQ_S1 : DQ_S0), smem_desc_sw128(q_base + qo, 16, 1024), smem_desc_sw128(kb + ko, 16, 1024),
                 IDESC_S, kk > 0);
          mma_ss(tmem + (w ? DQ_P1 : DQ_P0), smem_desc_sw128(do_base + qo, 16, 1024),
                 smem_desc_sw128(vb + ko, 16, 1024), IDESC_S, kk > 0);
        }
        tc_commit(&sdp_full[w]);
        return true;
      };
      if (ok && nblk > 0) ok = issue_sdp(0);
      if (ok && nblk > 1) ok = issue_sdp(1);
      for (int j = 0; ok && j < nblk; ++j) {
        const int w = j & 1, sk = j % NK;
        if (!mbar_wait(&p_full[w], (j >> 1) & 1, wc)) break;
        tc_fence_after();
        const uint32_t kb = k_base + sk * L::KB_BYTES;
#pragma unroll
        for (int kk = 0; kk < DQ_BN / 16; ++kk)
          mma_ts(tmem + DQ_ACC, tmem + (w ? DQ_P1 : DQ_P0) + kk * 8, smem_desc_sw128(kb + kk * 2048, KBOX, 1024),
                 IDESC_ACC, (j > 0 || kk > 0) ? 1u : 0u);
        tc_commit(&kv_empty[sk]);
        if (j + 2 < nblk) ok = issue_sdp(j + 2);
      }
      tc_commit(acc_done);
      mbar_wait_drain(acc_done, 0, wc);
    }
  } else {
    const int w = warp >> 2, quad = warp & 3, row = quad * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    const uint32_t tS = tmem + lane_addr + (w ? DQ_S1 : DQ_S0);
    const uint32_t tP = tmem + lane_addr + (w ? DQ_P1 : DQ_P0);
    const int qrow = min(q_row0 + row, g.N - 1);  // padding rows read a valid entry and are never stored
    const size_t qi = (size_t)bh * g.N + qrow;
    const float2 nl2 = make_float2(p.nlse2[qi], p.nlse2[qi]), nd2 = make_float2(p.ndelta[qi], p.ndelta[qi]);
    const float2 c2x2 = make_float2(p.c2, p.c2);
    bool ok = true;
    for (int j = w; j < nblk; j += 2) {
      const int it = j >> 1;
      ok = mbar_wait(&sdp_full[w], it & 1, wc);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const int valid = Lk - j * DQ_BN;
      const bool full_blk = valid >= DQ_BN;
      // straddling block over windows one tile apart (PAIR): 32-column chunks
      // of the key tile outside this warp's rows' window get dS = 0 (a chunk
      // never crosses a tile: s is a multiple of 64)
      unsigned drop = 0;
      if (PAIR && ks.rot) {
        const int x0 = straddle_excluded_start(p.gk.s, ks.ew, quad >> 1);
        int oq = (j * DQ_BN) % ks.run_len;
#pragma unroll
        for (int hh = 0; hh < DQ_BN / 32; ++hh) {
          if ((unsigned)(oq - x0) < (unsigned)p.gk.s) drop |= 1u << hh;
          oq += 32;
          if (oq >= ks.run_len) oq -= ks.run_len;
        }
      }
#pragma unroll
      for (int hh = 0; hh < DQ_BN / 32; ++hh) {
        const bool dropped = (drop >> hh) & 1u;
        if (PAIR && dropped) {  // chunk outside this warp's window: dS = 0, no exponentials
          const uint32_t z[16] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
          tmem_st16(tP + hh * 16, z);
          continue;
        }
        // one 32-column chunk at a time: S, dP and the packed dS stay in registers
        uint32_t sv[32], dv[32];
        tmem_ld32(tS + hh * 32, sv);
        tmem_ld32(tP + hh * 32, dv);
        tmem_wait_ld();
        uint32_t dk[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const float2 x = ffma2(make_float2(__uint_as_float(sv[2 * c]), __uint_as_float(sv[2 * c + 1])), c2x2, nl2);
          const float2 pp = make_float2(ex2(x.x), ex2(x.y));
          float2 o2 = fmul2(pp, fadd2(make_float2(__uint_as_float(dv[2 * c]), __uint_as_float(dv[2 * c + 1])), nd2));
          if (!full_blk) {
            const int cc = hh * 32 + 2 * c;
            if (cc >= valid) o2.x = 0.f;
            if (cc + 1 >= valid) o2.y = 0.f;
          }
          dk[c] = pack_bf16(o2.x, o2.y);
        }
        tmem_st16(tP + hh * 16, dk);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[w]);
    }
    if (ok && !*abort_flag) ok = mbar_wait(acc_done, 0, wc);
    ok = __all_sync(0xffffffffu, ok);
    tc_fence_after();
    if (ok && !*abort_flag) {
      const bool row_ok = row < q_valid;
      const uint32_t tAcc = tmem + lane_addr + DQ_ACC;
      const size_t grow = (size_t)bh * g.N + q_row0 + row;
#pragma unroll 1
      for (int c0 = (w * D) / 2; c0 < ((w + 1) * D) / 2; c0 += 32) {
        uint32_t x[32];
        tmem_ld32(tAcc + c0, x);
        tmem_wait_ld();
        if (row_ok) {
          float f[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) f[c] = __uint_as_float(x[c]) * p.scale;
          if (p.acc_out) {
            float4* dst = reinterpret_cast<float4*>(p.acc_out + grow * D + c0);
#pragma unroll
            for (int v4 = 0; v4 < 8; ++v4) dst[v4] = make_float4(f[4 * v4], f[4 * v4 + 1], f[4 * v4 + 2], f[4 * v4 + 3]);
          } else {
            if (p.acc_in) {
              const int prow = p.acc_pooled ? pooled_of_tiled(g, q_row0 + row) : 0;
              if (!dcheck(prow >= 0 && prow < g.Np, p.ctl.err_word)) continue;
              const size_t arow = p.acc_pooled ? (size_t)bh * g.Np + prow : grow;
              const float w = p.acc_pooled ? 1.f / (float)(g.pt * g.ph * g.pw) : 1.f;
              const float4* src = reinterpret_cast<const float4*>(p.acc_in + arow * D + c0);
#pragma unroll
              for (int v4 = 0; v4 < 8; ++v4) {
                const float4 a4 = __ldg(src + v4);
                f[4 * v4] += a4.x * w;
                f[4 * v4 + 1] += a4.y * w;
                f[4 * v4 + 2] += a4.z * w;
                f[4 * v4 + 3] += a4.w * w;
              }
            }
            uint4* dst = reinterpret_cast<uint4*>(p.dq + grow * D + c0);
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4)
              dst[v4] = make_uint4(pack_bf16(f[8 * v4], f[8 * v4 + 1]), pack_bf16(f[8 * v4 + 2], f[8 * v4 + 3]),
                                   pack_bf16(f[8 * v4 + 4], f[8 * v4 + 5]), pack_bf16(f[8 * v4 + 6], f[8 * v4 + 7]));
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == WARP_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

static int pow2_rows(int s, int cap) {
  int G = 1;
  while (G < cap && s % (G * 2) == 0) G *= 2;
  return G;
}

template <typename K>
static cudaError_t set_smem(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

// hk != NULL: hierarchical (coarse grid hk, factor = g's pool).  With global,
// the coarse-key pass (DKDV_HIER); without, the fine pass adding the coarse
// keys' fp32 gradients a.dkp / a.dvp through the medium pooling.
template <int D>
static cudaError_t launch_dkdv_d(const DevGeom& g, const BwdArgs& a, bool global, bool dual, cudaStream_t st,
                                 const DevGeom* hk = nullptr) {
  DkdvParams p;
  p.g = g;
  p.gk = g;
  p.gadd = g;
  p.cft = p.cfh = p.cfw = 1;
  p.hier_add = 0;
  p.mode = global ? DKDV_GLOBAL : DKDV_LOCAL;
  p.Gq = global ? 64 : pow2_rows(g.s, 64);
  p.kv_blocks_per_tile = (g.s + 127) / 128;
  // local keys: w-adjacent tiles of an odd multiple of 64 rows share their key
  // blocks (PairPlan), as the forward's query blocks
  p.pair = make_pair_plan(g, g.Nw, !global && !hk);
  p.Nk = global ? g.Np : g.N;
  if (hk && global) {
    p.gk = *hk;
    p.cft = g.pt;
    p.cfh = g.ph;
    p.cfw = g.pw;
    p.mode = DKDV_HIER;
    p.Gq = pow2_rows(g.s, 64);
    p.Nk = hk->N;
  } else if (hk) {  // fine keys: the streams stay on g, only the addend rows are coarse
    p.gadd = *hk;
    p.hier_add = 1;
  }
  p.scale = a.scale;
  p.c2 = a.scale * LOG2E;
  p.nlse2 = global ? a.nlse2_g : a.nlse2_l;
  p.ndelta = global ? a.ndelta_g : a.ndelta_l;
  p.dk = (__nv_bfloat16*)a.dk;
  p.dv = (__nv_bfloat16*)a.dv;
  p.dkp_out = global ? a.dkp : nullptr;
  p.dvp_out = global ? a.dvp : nullptr;
  p.dkp_in = (!global && dual) ? a.dkp : nullptr;
  p.dvp_in = (!global && dual) ? a.dvp : nullptr;
  p.ctl = current_ctl();
  const long long bh = (long long)g.B * g.heads;
  const bool pair = pair_plan_active(p.pair);
  const int blocks = p.mode == DKDV_GLOBAL ? (g.Np + 127) / 128
                     : p.mode == DKDV_HIER ? hk->n_tiles * p.kv_blocks_per_tile
                                           : (int)pair_plan_blocks(g, p.pair);
  if (bh == 0 || blocks == 0) return cudaSuccess;
  CUtensorMap tk, tv, tq, tdo;
  const char* err = nullptr;
  const void* kp = global ? a.kp : a.k;
  const void* vp = global ? a.vp : a.v;
  if (!make_tmap_rows(&tk, kp, D, p.Nk, bh, 128, &err) || !make_tmap_rows(&tv, vp, D, p.Nk, bh, 128, &err) ||
      !make_tmap_rows(&tq, a.q, D, g.N, bh, p.Gq, &err) || !make_tmap_rows(&tdo, a.dout, D, g.N, bh, p.Gq, &err))
    return cudaErrorInvalidValue;
  auto kernel = pair ? dkdv_kernel<D, true> : dkdv_kernel<D, false>;
  cudaError_t e = set_smem(kernel, DkdvSmem<D>::ALLOC);
  if (e != cudaSuccess) return e;
  kernel<<<dim3(blocks, (unsigned)bh), NTHREADS, DkdvSmem<D>::ALLOC, st>>>(tk, tv, tq, tdo, p);
  return cudaGetLastError();
}

// hk != NULL: the coarse-key pass of the hierarchical branch (DQ_HIER) into
// the fp32 a.dq_acc; keys a.kp / a.vp in hk's tile-major order.
template <int D>
static cudaError_t launch_dq_d(const DevGeom& g, const BwdArgs& a, bool global, bool add_acc, cudaStream_t st,
                               const DevGeom* hk = nullptr) {
  DqParams p;
  p.g = g;
  p.gk = hk ? *hk : g;
  p.cft = hk ? g.pt : 1;
  p.cfh = hk ? g.ph : 1;
  p.cfw = hk ? g.pw : 1;
  p.mode = global ? DQ_GLOBAL : hk ? DQ_HIER : DQ_LOCAL;
  int G0 = DQ_BN;  // largest multiple of 8 dividing both the key block and the tile volume
  while (G0 > 8 && (DQ_BN % G0 != 0 || g.s % G0 != 0)) G0 -= 8;
  p.G0 = G0;
  p.q_blocks_per_tile = (g.s + 127) / 128;
  // local and hierarchical passes: w-adjacent tiles of an odd multiple of 64
  // rows share their query blocks (PairPlan), as in the forward
  p.pair = make_pair_plan(g, p.gk.Nw, !global);
  const bool pair = pair_plan_active(p.pair);
  p.scale = a.scale;
  p.c2 = a.scale * LOG2E;
  p.nlse2 = global ? a.nlse2_g : a.nlse2_l;
  p.ndelta = global ? a.ndelta_g : a.ndelta_l;
  p.acc_in = (!global && !hk && add_acc) ? a.dq_acc : nullptr;
  p.acc_pooled = a.dq_acc_pooled ? 1 : 0;
  p.acc_out = (global || hk) ? a.dq_acc : nullptr;
  p.dq = (__nv_bfloat16*)a.dq;
  p.ctl = current_ctl();
  const long long bh = (long long)g.B * g.heads;
  const int blocks = global ? (g.N + 127) / 128 : (int)pair_plan_blocks(g, p.pair);
  if (bh == 0 || blocks == 0) return cudaSuccess;
  CUtensorMap tq, tdo, tk, tv;
  const char* err = nullptr;
  const void* kk = (global || hk) ? a.kp : a.k;
  const void* vv = (global || hk) ? a.vp : a.v;
  const long long nk = global ? g.Np : hk ? hk->N : g.N;
  const int G = global ? DQ_BN : p.G0;
  if (!make_tmap_rows(&tq, a.q, D, g.N, bh, 128, &err) || !make_tmap_rows(&tdo, a.dout, D, g.N, bh, 128, &err) ||
      !make_tmap_rows(&tk, kk, D, nk, bh, G, &err) || !make_tmap_rows(&tv, vv, D, nk, bh, G, &err))
    return cudaErrorInvalidValue;
  auto kernel = pair ? dq_kernel<D, true> : dq_kernel<D, false>;
  cudaError_t e = set_smem(kernel, DqSmem<D>::ALLOC);
  if (e != cudaSuccess) return e;
  kernel<<<dim3(blocks, (unsigned)bh), NTHREADS, DqSmem<D>::ALLOC, st>>>(tq, tdo, tk, tv, p);
  return cudaGetLastError();
}

}  // namespace bwd

// Blocks per batch*head slice of the preprocess: the whole launch one wave of
// 8 resident 256-thread blocks per SM, each block's loop striding over its
// slice (a launch of several partial waves left the HBM idle in its tail).
static int preprocess_blocks(const DevGeom& g, long long bh) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int rows_per_block = 256 / (g.d / 8);
  long long blocks = (long long)sms * 8 / (bh > 0 ? bh : 1);
  const long long need = (g.N + rows_per_block - 1) / rows_per_block;
  if (blocks > need) blocks = need;
  return (int)(blocks < 1 ? 1 : blocks);
}

cudaError_t launch_bwd_preprocess(const DevGeom& g, const BwdArgs& a, bool dual, cudaStream_t st) {
  const long long bh = (long long)g.B * g.heads;
  if (bh == 0 || g.N == 0) return cudaSuccess;
  if (dual && a.dg) {
    cudaError_t e = cudaMemsetAsync(a.dg, 0, sizeof(float) * g.heads, st);
    if (e != cudaSuccess) return e;
  }
  bwd::PreArgs pa;
  pa.dout = (const uint4*)a.dout;
  pa.o_l = (const uint4*)a.o_l;
  pa.o_g = dual ? (const uint4*)a.o_g : nullptr;
  pa.lse_l = a.lse_l;
  pa.lse_g = dual ? a.lse_g : nullptr;
  pa.ndelta_l = a.ndelta_l;
  pa.ndelta_g = dual ? a.ndelta_g : nullptr;
  pa.nlse2_l = a.nlse2_l;
  pa.nlse2_g = dual ? a.nlse2_g : nullptr;
  pa.dg = dual ? a.dg : nullptr;
  pa.gvec = dual ? a.g : nullptr;
  pa.vpr = g.d / 8;
  pa.N = g.N;
  pa.heads = g.heads;
  bwd::bwd_preprocess_kernel<<<dim3(preprocess_blocks(g, bh), (unsigned)bh), 256, 0, st>>>(pa);
  return cudaGetLastError();
}

cudaError_t launch_preprocess_branch(const DevGeom& g, const void* dout, const void* o, const float* lse,
                                     const float* gvec, float* ndelta, float* nlse2, cudaStream_t st) {
  const long long bh = (long long)g.B * g.heads;
  if (bh == 0 || g.N == 0) return cudaSuccess;
  bwd::PreArgs pa;
  pa.dout = (const uint4*)dout;
  pa.o_l = (const uint4*)o;
  pa.o_g = nullptr;
  pa.lse_l = lse;
  pa.lse_g = nullptr;
  pa.ndelta_l = ndelta;
  pa.ndelta_g = nullptr;
  pa.nlse2_l = nlse2;
  pa.nlse2_g = nullptr;
  pa.dg = nullptr;
  pa.gvec = gvec;
  pa.vpr = g.d / 8;
  pa.N = g.N;
  pa.heads = g.heads;
  bwd::bwd_preprocess_kernel<<<dim3(preprocess_blocks(g, bh), (unsigned)bh), 256, 0, st>>>(pa);
  return cudaGetLastError();
}

cudaError_t launch_bwd_dkdv_global(const DevGeom& g, const BwdArgs& a, cudaStream_t st) {
  if (g.d == 128) return bwd::launch_dkdv_d<128>(g, a, true, true, st);
  if (g.d == 64) return bwd::launch_dkdv_d<64>(g, a, true, true, st);
  return cudaErrorInvalidValue;
}

cudaError_t launch_bwd_dkdv_local(const DevGeom& g, const BwdArgs& a, bool dual, cudaStream_t st) {
  if (g.d == 128) return bwd::launch_dkdv_d<128>(g, a, false, dual, st);
  if (g.d == 64) return bwd::launch_dkdv_d<64>(g, a, false, dual, st);
  return cudaErrorInvalidValue;
}

cudaError_t launch_bwd_dq_global(const DevGeom& g, const BwdArgs& a, cudaStream_t st) {
  if (g.d == 128) return bwd::launch_dq_d<128>(g, a, true, false, st);
  if (g.d == 64) return bwd::launch_dq_d<64>(g, a, true, false, st);
  return cudaErrorInvalidValue;
}

cudaError_t launch_bwd_dkdv_hier(const DevGeom& g, const DevGeom& gc, const BwdArgs& a, bool coarse_keys,
                                 cudaStream_t st) {
  if (g.d == 128) return bwd::launch_dkdv_d<128>(g, a, coarse_keys, !coarse_keys, st, &gc);
  if (g.d == 64) return bwd::launch_dkdv_d<64>(g, a, coarse_keys, !coarse_keys, st, &gc);
  return cudaErrorInvalidValue;
}

cudaError_t launch_bwd_dq_hier(const DevGeom& g, const DevGeom& gc, const BwdArgs& a, cudaStream_t st) {
  if (g.d == 128) return bwd::launch_dq_d<128>(g, a, false, false, st, &gc);
  if (g.d == 64) return bwd::launch_dq_d<64>(g, a, false, false, st, &gc);
  return cudaErrorInvalidValue;
}

cudaError_t launch_bwd_dq(const DevGeom& g, const BwdArgs& a, bool dual, cudaStream_t st) {
  if (g.d == 128) return bwd::launch_dq_d<128>(g, a, false, dual, st);
  if (g.d == 64) return bwd::launch_dq_d<64>(g, a, false, dual, st);
  return cudaErrorInvalidValue;
}

}  // namespace vattn

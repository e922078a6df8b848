// lf_tc_bwd.cu -- tensor-core (tcgen05 / TMEM / TMA) backward of Longformer
// attention, bf16 / f16 inputs, fp32 accumulation, for the loss L = sum(o * dO).
//
// With P the attention probabilities (recomputed from the forward's
// log-normaliser, never stored), dP = dO V^T, D_i = rowsum(dO_i * O_i) and
// dS = P * (dP - D) * scale:   dQ = dS K,  dK = dS^T Q,  dV = P^T dO
// (the softmax Jacobian; global rows use Q_g / K_g / V_g, local rows
// Q_s / K_s / V_s, segmentfault page sections 全局注意力 / 全局注意力的线性投影).
//
// Two work-item kinds run on the same tensor-core pipeline, one 128-row
// block of a residue sub-sequence per CTA (dilated heads use the forward's
// residue tensor-map views):
//  * mode Q  (rows = local queries):  per key tile  S = Q K^T, dP = dO V^T;
//             the softmax warps form dS (TMEM) and the MMA warp accumulates
//             dQ += dS K.  Key tiles are the band tiles of the block and the
//             global-column tiles (global keys outside each row's window).
//             Writes dQ_s (zero for global and mask-0 rows).
//  * mode KV (rows = keys):  per band query tile  S^T = K Q^T, dP^T = V dO^T;
//             the softmax warps form P^T and dS^T (TMEM) from the queries'
//             log-normaliser and D (staged per tile in shared memory by the
//             producer warp; +inf log-normaliser for columns that are not
//             local queries, so their probability is 0), and the MMA warp
//             accumulates dV += P^T dO, dK += dS^T Q.  Writes the band part of
//             dK_s, dV_s (the global-column part of the global keys is added
//             afterwards by lf_bwd_gcol_*).
// Column tiles are 64 wide (keys in mode Q, queries in mode KV).  Roles per
// CTA (192 threads, 256 TMEM columns, ~98 KB of shared memory: two CTAs per
// SM, so one CTA's MMA round trip overlaps the other's exponentials): warps
// 0-3 form P / dS (one TMEM lane = one row), warp 4 issues TMA loads (row
// operands once, column operands into a 4-stage ring), warp 5 issues the
// MMAs.  TMEM: S [0,64), dP [64,128), acc0 [128,192) (dQ or dV), acc1
// [192,256) (dK).  The 16-bit A operands of the accumulating products are
// written over the columns they were computed from, chunk by chunk once
// read: dS (mode Q) or P^T (mode KV) into S's first 32 columns, dS^T into
// dP's.  The next tile's S and dP are issued after those products by the
// same thread, and tcgen05 operations of one thread run in order, so they
// overwrite the A operands only after they have been read.
// Every mbarrier wait is bounded (status LF_ERR_DEVICE_TIMEOUT on expiry).
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <map>
#include <utility>

#include "lf_ptx.cuh"
#include "lf_tc.cuh"

#define LF_BW_THREADS 192
#define LF_BW_NS 4
#define LF_BW_BK 64  // columns (keys / queries) per column tile
#define LF_BW_MAX_MAPS 192  // kernel parameters may take up to 32 KB
#define LF_BW_MAX_SEG 96
#define LF_BW_ROWS_PER_CHUNK 64  // keys per chunk of the global-key pass (dK_g, dV_g, dQ_g)
#define LF_BW_GKEY_EB 4          // global rows per reduction of the global-key pass (256 / 64 outputs)
#define LF_BW_GCOL_ROWS 256      // rows per chunk of the global-column pass

#define LF_BW_R0 0
#define LF_BW_R1 16384
#define LF_BW_CST (LF_BW_BK * 128 * 2)  // one column stage: two 64-row tiles
#define LF_BW_C0(s) (32768 + (s)*LF_BW_CST)
#define LF_BW_C1(s) (32768 + (s)*LF_BW_CST + LF_BW_BK * 128)
#define LF_BW_VEC(s) (32768 + LF_BW_NS * LF_BW_CST + (s)*(2 * LF_BW_BK * 4))
#define LF_BW_BAR (32768 + LF_BW_NS * LF_BW_CST + LF_BW_NS * 2 * LF_BW_BK * 4)
#define LF_BW_SMEM (LF_BW_BAR + 256)
static_assert(2 * (LF_BW_SMEM + 1024) <= 233472, "two CTAs per SM");

#define LF_BT_S 0
#define LF_BT_DP 64
#define LF_BT_ACC0 128
#define LF_BT_ACC1 192
#define LF_BT_COLS 256

struct LfBwParams {
  CUtensorMap maps[LF_BW_MAX_MAPS];  // per residue view: q, k, v, dO (128-row boxes), the same
                                     // with 64-row boxes; then ks_c, vs_c
  LfDev dev;
  LfTcSeg seg[LF_BW_MAX_SEG];
  int nseg, per_batch, gbox, map_ksc, map_vsc;
  const float *lse;
  const float *delta;
  void *dq_out, *dk_out, *dv_out;  // dQ_s (mode Q); dK_s, dV_s (mode KV)
};

// Work item (shared decode for every role).
struct LfBwItem {
  int b, h, d, rho, cnt, row0, map, nband, nglob, T, ng;
};

__device__ __forceinline__ void lf_bw_decode(const LfBwParams &P, int idx, int modeq,
                                             LfBwItem &it) {
  const LfDev &D = P.dev;
  it.b = idx / P.per_batch;
  int rem = idx - it.b * P.per_batch;
  int s = 0;
  while (s + 1 < P.nseg && rem >= P.seg[s + 1].start) s++;
  const LfTcSeg &sg = P.seg[s];
  rem -= sg.start;
  it.h = sg.h0 + rem / sg.nqb;
  it.row0 = (rem % sg.nqb) * LF_BQ;
  it.d = sg.d;
  it.rho = sg.rho;
  it.cnt = sg.cnt;
  it.map = sg.map;
  it.nband = lf_band_tiles_w<LF_BW_BK>(D.r, D.causal);
  const int32_t *bi = D.binfo + (size_t)it.b * LF_BI_WORDS;
  it.ng = bi[LF_BI_NG];
  it.nglob = 0;
  if (modeq && it.ng > 0) {
    bool need = true;
    if (it.d == 1 && !D.causal) {
      const int tlast = min(it.row0 + LF_BQ - 1, it.cnt - 1);
      if (bi[LF_BI_GMIN] >= tlast - D.r && bi[LF_BI_GMAX] <= it.row0 + D.r) need = false;
    }
    it.nglob = need ? (it.ng + LF_BW_BK - 1) / LF_BW_BK : 0;
  }
  it.T = it.nband + it.nglob;
}

// first column-operand row of band tile u
__device__ __forceinline__ int lf_bw_tile_row(const LfDev &D, const LfBwItem &it, int modeq, int u) {
  if (modeq || !D.causal) return it.row0 - D.r + LF_BW_BK * u;
  return it.row0 + LF_BW_BK * u;  // causal, rows = keys: queries t in [j, j + r]
}

// One work item (a 128-row block) of mode kModeQ.
template <int kF16, int kModeQ>
__device__ __forceinline__ void lf_tc_bwd_item(const LfBwParams &P, int item, uint8_t *lf_bw_smem) {
  const uint32_t sbase = lf_smem(lf_bw_smem);
  if (sbase & 1023u) {
    if (threadIdx.x == 0) lf_set_status(P.dev.status, LF_ERR_UNSUPPORTED, 9001);
    return;
  }
  uint8_t *gbase = lf_bw_smem;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const LfDev &D = P.dev;
  const int n = D.n;
  LfBwItem it;
  lf_bw_decode(P, item, kModeQ, it);
  const int T = it.T;

  const uint32_t bar = sbase + LF_BW_BAR;
  const uint32_t row_full = bar, s_full = bar + 8, ds_full = bar + 16, o_full = bar + 32,
                 end_bar = bar + 40;
  const uint32_t col_full0 = bar + 48, col_empty0 = bar + 48 + 8 * LF_BW_NS;
  uint32_t *tmem_slot = (uint32_t *)(gbase + LF_BW_BAR + 192);
  volatile int *abort_flag = (volatile int *)(gbase + LF_BW_BAR + 196);  // [2]: flag, wait limit

  if (threadIdx.x == 0) {
    lf_mbar_init(row_full, 1);
    lf_mbar_init(s_full, 1);
    lf_mbar_init(ds_full, 4);
    lf_mbar_init(o_full, 1);
    lf_mbar_init(end_bar, 1);
    for (int s = 0; s < LF_BW_NS; s++) {
      lf_mbar_init(col_full0 + 8 * s, kModeQ ? 1 : 2);
      lf_mbar_init(col_empty0 + 8 * s, 1);
    }
    abort_flag[0] = 0;
    abort_flag[1] = P.dev.wait_us;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 5) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     lf_smem(tmem_slot)),
                 "r"(LF_BT_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  lf_tc_fence_before();
  __syncthreads();
  lf_tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const size_t bh = (size_t)it.b * D.H + it.h;
  const int32_t *mrow = D.mask + (size_t)it.b * n;

  if (warp == 4) {
    // ================================================== TMA producer (+ column vectors)
    const CUtensorMap *mq = &P.maps[it.map], *mk = &P.maps[it.map + 1], *mv = &P.maps[it.map + 2],
                      *mdo = &P.maps[it.map + 3];
    // the same views with 64-row boxes, for the column tiles
    const CUtensorMap *cq = &P.maps[it.map + 4], *ck = &P.maps[it.map + 5], *cv = &P.maps[it.map + 6],
                      *cdo = &P.maps[it.map + 7];
    if (lane == 0) {
      lf_mbar_expect_tx(row_full, 32768);
      lf_tma_load4(sbase + LF_BW_R0, kModeQ ? mq : mk, row_full, 0, it.row0, it.h, it.b);
      lf_tma_load4(sbase + LF_BW_R1, kModeQ ? mdo : mv, row_full, 0, it.row0, it.h, it.b);
    }
    int issued = 0;
    for (int t = 0; t < T; t++) {
      const int s = t % LF_BW_NS;
      if (t >= LF_BW_NS &&
          !lf_wait_warp(col_empty0 + 8 * s, ((t / LF_BW_NS) & 1) ^ 1, abort_flag, D.status, 21))
        break;
      int row;
      const CUtensorMap *c0, *c1;
      uint32_t bytes;
      if (t < it.nband) {
        row = lf_bw_tile_row(D, it, kModeQ, t);
        c0 = kModeQ ? ck : cq;
        c1 = kModeQ ? cv : cdo;
        bytes = 2 * LF_BW_BK * 128;
      } else {
        row = (t - it.nband) * LF_BW_BK;
        c0 = &P.maps[P.map_ksc];
        c1 = &P.maps[P.map_vsc];
        bytes = 2 * P.gbox * 128;
      }
      if (!kModeQ) {
        // per-column (query) log-normaliser in log2 units and D; +inf marks
        // columns that are not local queries (probability 0)
        float *lse2 = (float *)(gbase + LF_BW_VEC(s));
        float *dv = lse2 + LF_BW_BK;
#pragma unroll
        for (int k = 0; k < LF_BW_BK / 32; k++) {
          const int c = lane + 32 * k, tq = row + c;
          float l2 = INFINITY, dd = 0.f;
          if (tq >= 0 && tq < it.cnt) {
            const int pos = it.rho + tq * it.d;
            if (mrow[pos] == 1) {
              l2 = P.lse[bh * n + pos] * LF_LOG2E;
              dd = P.delta[bh * n + pos];
            }
          }
          lse2[c] = l2;
          dv[c] = dd;
        }
        __syncwarp();
      }
      if (lane == 0) {
        lf_mbar_expect_tx(col_full0 + 8 * s, bytes);
        lf_tma_load4(sbase + LF_BW_C0(s), c0, col_full0 + 8 * s, 0, row, it.h, it.b);
        lf_tma_load4(sbase + LF_BW_C1(s), c1, col_full0 + 8 * s, 0, row, it.h, it.b);
        if (!kModeQ) lf_mbar_arrive(col_full0 + 8 * s);
      }
      issued = t + 1;
    }
    if (*abort_flag && lane == 0) {
      for (int t = max(0, issued - LF_BW_NS); t < issued; t++)
        lf_wait_drain(col_full0 + 8 * (t % LF_BW_NS), (t / LF_BW_NS) & 1, D.status, 22);
    }
  } else if (warp == 5) {
    // ================================================== MMA issuer
    // the whole warp waits; one elected lane issues each phase
    const uint64_t dr0 = lf_sdesc(sbase + LF_BW_R0, 16, 1024);
    const uint64_t dr1 = lf_sdesc(sbase + LF_BW_R1, 16, 1024);
    const uint64_t dc0 = lf_sdesc(sbase + LF_BW_C0(0), 16, 1024);  // K-major view
    const uint64_t dc0mn = lf_sdesc(sbase + LF_BW_C0(0), 0, 1024);  // MN-major view
    const uint64_t dc1 = lf_sdesc(sbase + LF_BW_C1(0), 16, 1024);
    const uint64_t dc1mn = lf_sdesc(sbase + LF_BW_C1(0), 0, 1024);
    const uint32_t id_acc = lf_idesc(kF16, 64, 1);
    const int ngk = (it.ng + 15) / 16 * 16;
    auto ncols = [&](int t) {
      return t < it.nband ? LF_BW_BK : min(LF_BW_BK, ngk - (t - it.nband) * LF_BW_BK);
    };
    // S = R0 C0^T and dP = R1 C1^T of column tile t -> s_full
    auto issue_s = [&](int t) {
      const uint64_t so = (uint64_t)((t % LF_BW_NS) * (LF_BW_CST >> 4));
      lf_mma_s2_phase(tmem + LF_BT_S, dr0, dc0 + so, tmem + LF_BT_DP, dr1, dc1 + so,
                      lf_idesc(kF16, ncols(t), 0), s_full);
    };
    bool ok = lf_wait_warp(row_full, 0, abort_flag, D.status, 23) &&
              lf_wait_warp(col_full0, 0, abort_flag, D.status, 24);
    if (ok) {
      lf_tc_fence_after();
      issue_s(0);
      for (int t = 0; t < T; t++) {
        if (!lf_wait_warp(ds_full, t & 1, abort_flag, D.status, 25)) break;
        lf_tc_fence_after();
        const uint64_t so = (uint64_t)((t % LF_BW_NS) * (LF_BW_CST >> 4));
        const uint32_t kmask = (1u << (ncols(t) / 16)) - 1u;
        const uint32_t acc0 = t > 0 ? 1u : 0u;
        const uint32_t last = t + 1 == T ? o_full : 0u;
        if (kModeQ) {
          // dQ += dS K   (dS packed in S's columns; K tile as the MN-major B operand)
          lf_mma_ts_phase(tmem + LF_BT_ACC0, tmem + LF_BT_S, dc0mn + so, 2048 >> 4, id_acc, kmask,
                          acc0, col_empty0 + 8 * (t % LF_BW_NS), last, 0u);
        } else {
          // dV += P^T dO ; dK += dS^T Q   (P^T in S's columns, dS^T in dP's)
          lf_mma_ts_phase(tmem + LF_BT_ACC0, tmem + LF_BT_S, dc1mn + so, 2048 >> 4, id_acc, kmask,
                          acc0, 0u, 0u, 0u);
          lf_mma_ts_phase(tmem + LF_BT_ACC1, tmem + LF_BT_DP, dc0mn + so, 2048 >> 4, id_acc, kmask,
                          acc0, col_empty0 + 8 * (t % LF_BW_NS), last, 0u);
        }
        // the next tile's S and dP, issued after the products that read this
        // tile's A operands out of the same columns
        if (t + 1 < T) {
          const int s2 = (t + 1) % LF_BW_NS;
          if (!lf_wait_warp(col_full0 + 8 * s2, ((t + 1) / LF_BW_NS) & 1, abort_flag, D.status, 26))
            break;
          lf_tc_fence_after();
          issue_s(t + 1);
        }
      }
    }
    lf_commit_w(end_bar);
    lf_wait_drain(end_bar, 0, D.status, 27);  // also after an abort: TMEM is freed after this
    __syncwarp();
  } else {
    // ================================================== P / dS warps (0..3)
    const int q = warp * 32 + lane;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const uint32_t tS = tmem + lane_off + LF_BT_S, tDP = tmem + lane_off + LF_BT_DP;
    const float sl2 = D.scale_log2, scale = D.scale;
    const int trow = it.row0 + q;
    int pos = 0, code = 0;
    if (trow < it.cnt) {
      pos = it.rho + trow * it.d;
      code = mrow[pos];
    }
    // mode Q: local query rows; mode KV: valid key rows
    const bool active = kModeQ ? (code == 1) : (trow < it.cnt && code != 0);
    float lse2 = 0.f, dd = 0.f;
    if (kModeQ && active) {
      lse2 = P.lse[bh * n + pos] * LF_LOG2E;
      dd = P.delta[bh * n + pos];
    }
    const bool padded = D.binfo[(size_t)it.b * LF_BI_WORDS + LF_BI_NVALID] < n;
    const int32_t *gl = D.gidx + (size_t)it.b * D.G;
    int e_lo = 0, e_hi = 0;
    if (kModeQ && it.nglob > 0 && active) {
      const int32_t *gr = D.grank + (size_t)it.b * (n + 1);
      e_lo = gr[max(pos - D.r * it.d, 0)];
      e_hi = gr[min((D.causal ? pos : pos + D.r * it.d) + 1, n)];
    }
    bool alive = true;
    for (int t = 0; t < T && alive; t++) {
      if (!lf_wait_warp(s_full, t & 1, abort_flag, D.status, 28)) {
        alive = false;
        break;
      }
      lf_tc_fence_after();
      constexpr int NC = LF_BW_BK / 32;  // 32-column chunks per tile
      uint32_t w[NC];
      const int s = t % LF_BW_NS;
      if (t < it.nband) {
        const int kb = lf_bw_tile_row(D, it, kModeQ, t);
        int lo, hi;
        lf_band_cols_w<LF_BW_BK>(q, t, D.r, D.causal, lo, hi);
        lo = max(lo, -kb);  // column operand rows exist on [0, cnt)
        hi = min(hi, it.cnt - 1 - kb);
        if (!active) hi = -1;
#pragma unroll
        for (int cc = 0; cc < NC; cc++) w[cc] = lf_range_bits(lo, hi, 32 * cc);
        if (kModeQ && padded) {
#pragma unroll
          for (int cc = 0; cc < NC; cc++) {
            const int tk = kb + 32 * cc + lane;
            const bool okk = tk >= 0 && tk < it.cnt && mrow[it.rho + tk * it.d] != 0;
            w[cc] &= __ballot_sync(0xffffffffu, okk);
          }
        }
      } else {
        const int gbs = (t - it.nband) * LF_BW_BK;
        const int hi = active ? min(LF_BW_BK - 1, it.ng - 1 - gbs) : -1;
#pragma unroll
        for (int cc = 0; cc < NC; cc++) {
          uint32_t inwin = lf_range_bits(e_lo - gbs, e_hi - 1 - gbs, 32 * cc);
          if (it.d > 1) {
            const int e = gbs + 32 * cc + lane;
            const bool res = e < it.ng && (gl[e] - it.rho) % it.d == 0;
            inwin &= __ballot_sync(0xffffffffu, res);
          }
          w[cc] = lf_range_bits(0, hi, 32 * cc) & ~inwin;
        }
      }
      if (!kModeQ) {
        // the per-column vectors of stage s were written by the producer
        // warp before it arrived on col_full(s): observe that phase here too
        if (!lf_wait_warp(col_full0 + 8 * s, (t / LF_BW_NS) & 1, abort_flag, D.status, 31)) {
          alive = false;
          break;
        }
      }
      const float *clse2 = (const float *)(gbase + LF_BW_VEC(s));
      const float *cdd = clse2 + LF_BW_BK;
#pragma unroll
      for (int cc = 0; cc < NC; cc++) {
        uint32_t ds_w[16], p_w[16];
        if (__any_sync(0xffffffffu, w[cc] != 0u)) {
          // S and dP of the chunk in flight together, one wait
          uint32_t x[32], y[32];
          lf_tmem_ld32_nowait(tS + 32 * cc, x);
          lf_tmem_ld32_nowait(tDP + 32 * cc, y);
          lf_tmem_wait_ld_regs(x);
          lf_tmem_pin_regs(y);
          const uint32_t wc = w[cc];
#pragma unroll
          for (int k4 = 0; k4 < 32; k4 += 4) {
            // the columns' log-normalisers and D (mode KV), four per shared-memory load
            float4 l4 = make_float4(lse2, lse2, lse2, lse2), d4 = make_float4(dd, dd, dd, dd);
            if (!kModeQ) {
              l4 = *reinterpret_cast<const float4 *>(clse2 + 32 * cc + k4);
              d4 = *reinterpret_cast<const float4 *>(cdd + 32 * cc + k4);
            }
            const float lv[4] = {l4.x, l4.y, l4.z, l4.w}, dv[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
            for (int u = 0; u < 4; u += 2) {
              const int k = k4 + u;
              float p0 = 0.f, p1 = 0.f, g0 = 0.f, g1 = 0.f;
              if ((wc >> k) & 1u) {
                p0 = lf_ex2(fmaf(__uint_as_float(x[k]), sl2, -lv[u]));
                g0 = p0 * (__uint_as_float(y[k]) - dv[u]) * scale;
              }
              if ((wc >> (k + 1)) & 1u) {
                p1 = lf_ex2(fmaf(__uint_as_float(x[k + 1]), sl2, -lv[u + 1]));
                g1 = p1 * (__uint_as_float(y[k + 1]) - dv[u + 1]) * scale;
              }
              ds_w[k / 2] = lf_pack2<kF16>(g0, g1);
              p_w[k / 2] = lf_pack2<kF16>(p0, p1);
            }
          }
        } else {
#pragma unroll
          for (int k = 0; k < 16; k++) ds_w[k] = p_w[k] = 0u;
        }
        // packed over columns [16cc, 16cc + 16) of S (and dP): chunk cc's
        // scores are in registers and chunk cc+1's columns lie beyond them
        if (kModeQ) {
          lf_tmem_st16(tS + 16 * cc, ds_w);
        } else {
          lf_tmem_st16(tS + 16 * cc, p_w);
          lf_tmem_st16(tDP + 16 * cc, ds_w);
        }
      }
      if (!alive) break;
      lf_tmem_wait_st();
      lf_tc_fence_before();
      __syncwarp();
      if (lane == 0) lf_mbar_arrive(ds_full);
    }
    // ---- epilogue: accumulators -> gradient rows
    if (alive && lf_wait_warp(o_full, 0, abort_flag, D.status, 30)) {
      lf_tc_fence_after();
      // TMEM loads are warp-collective: every lane loads, only rows that exist store
      const bool store = trow < it.cnt;
      const size_t orow = bh * n + pos;
      const float keep = active ? 1.f : 0.f;
#pragma unroll
      for (int which = 0; which < (kModeQ ? 1 : 2); which++) {
        float a[32], c2[32];
        lf_tmem_ld32(tmem + lane_off + (which ? LF_BT_ACC1 : LF_BT_ACC0), a);
        lf_tmem_ld32(tmem + lane_off + (which ? LF_BT_ACC1 : LF_BT_ACC0) + 32, c2);
        if (!store) continue;
        void *outp = kModeQ ? P.dq_out : (which ? P.dk_out : P.dv_out);
        uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<uint16_t *>(outp) + orow * LF_HD);
#pragma unroll
        for (int k = 0; k < 4; k++) {
          uint4 u;
          u.x = lf_pack2<kF16>(a[8 * k + 0] * keep, a[8 * k + 1] * keep);
          u.y = lf_pack2<kF16>(a[8 * k + 2] * keep, a[8 * k + 3] * keep);
          u.z = lf_pack2<kF16>(a[8 * k + 4] * keep, a[8 * k + 5] * keep);
          u.w = lf_pack2<kF16>(a[8 * k + 6] * keep, a[8 * k + 7] * keep);
          dst[k] = u;
          uint4 v;
          v.x = lf_pack2<kF16>(c2[8 * k + 0] * keep, c2[8 * k + 1] * keep);
          v.y = lf_pack2<kF16>(c2[8 * k + 2] * keep, c2[8 * k + 3] * keep);
          v.z = lf_pack2<kF16>(c2[8 * k + 4] * keep, c2[8 * k + 5] * keep);
          v.w = lf_pack2<kF16>(c2[8 * k + 6] * keep, c2[8 * k + 7] * keep);
          dst[4 + k] = v;
        }
      }
    }
  }

  lf_tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    lf_tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(LF_BT_COLS)
                 : "memory");
  }
}

// Both modes in one launch: blocks [0, items) are mode KV (dK_s, dV_s),
// blocks [items, 2 items) mode Q (dQ_s).  The two are independent (both
// read the forward's lse and the row deltas), so their CTAs share the SMs
// and fill each other's tails.
template <int kF16>
__global__ void __launch_bounds__(LF_BW_THREADS, 2)
    lf_tc_bwd_kernel(const __grid_constant__ LfBwParams P) {
  extern __shared__ __align__(1024) uint8_t lf_bw_smem[];
  const int items = P.dev.B * P.per_batch;
  if ((int)blockIdx.x < items)
    lf_tc_bwd_item<kF16, 0>(P, blockIdx.x, lf_bw_smem);
  else
    lf_tc_bwd_item<kF16, 1>(P, blockIdx.x - items, lf_bw_smem);
}

// ============================================== global-token parts (CUDA cores)

// Global-column part of dK_s / dV_s: a global key g is attended by every
// local row, by its window or by its global column (union); the band kernel
// covered the window, this pass the rows whose window misses g.  One block of
// 256 threads per (b, h, global e, chunk of LF_BW_GCOL_ROWS rows),
// grid-strided: a lane group (64 / N lanes, 16 bytes of a row each) per row,
// the groups' sums added in a fixed order into the chunk's partial, which
// lf_bwd_gcol_reduce adds up.
template <typename T>
__global__ void __launch_bounds__(256, 2)
    lf_bwd_gcol_kernel(LfDev P, const T *qs, const T *ks, const T *vs, const float *lse,
                       const T *dO, const float *delta, float *part, int nch) {
  constexpr int N = LfVec<T>::N, TPR = LF_HD / N, GPB = 256 / TPR;
  __shared__ float s_red[8][2 * LF_HD];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int grp = threadIdx.x / TPR, pi = threadIdx.x % TPR;
  const long long units = (long long)P.B * P.H * P.G * nch;
  for (long long un = blockIdx.x; un < units; un += gridDim.x) {
    const int c = (int)(un % nch);
    const long long be = un / nch;
    const int e = (int)(be % P.G);
    const long long bh = be / P.G;
    const int h = (int)(bh % P.H), b = (int)(bh / P.H), d = P.dil[h], n = P.n;
    const int ng = P.binfo[(size_t)b * LF_BI_WORDS + LF_BI_NG];
    float ak[N], av[N];
#pragma unroll
    for (int k = 0; k < N; k++) ak[k] = av[k] = 0.f;
    if (e < ng) {
      const int g = P.gidx[(size_t)b * P.G + e];
      const int32_t *m = P.mask + (size_t)b * n;
      const size_t base = (size_t)bh * n * LF_HD + pi * N;
      float kx[N], vx[N];
      LfVec<T>::ld(ks + base + (size_t)g * LF_HD, kx);
      LfVec<T>::ld(vs + base + (size_t)g * LF_HD, vx);
      const int i0 = c * LF_BW_GCOL_ROWS, i1 = min(n, i0 + LF_BW_GCOL_ROWS);
      // four row groups per round: every load of the round is issued before
      // any of its arithmetic (none waits on a mask test)
      for (int rr = 0; rr < LF_BW_GCOL_ROWS; rr += 4 * GPB) {
        float q[4][N], go[4][N], lse_i[4], dl_i[4];
        int mi[4];
#pragma unroll
        for (int u = 0; u < 4; u++) {
          const int i = i0 + rr + u * GPB + grp;
          const int ic = i < i1 ? i : i1 - 1;
          LfVec<T>::ld(qs + base + (size_t)ic * LF_HD, q[u]);
          LfVec<T>::ld(dO + base + (size_t)ic * LF_HD, go[u]);
          const size_t ir = (size_t)bh * n + ic;
          mi[u] = m[ic];
          lse_i[u] = lse[ir];
          dl_i[u] = delta[ir];
        }
#pragma unroll
        for (int u = 0; u < 4; u++) {
          const int i = i0 + rr + u * GPB + grp;
          float s = 0.f, dp = 0.f;
#pragma unroll
          for (int k = 0; k < N; k++) {
            s += q[u][k] * kx[k];
            dp += go[u][k] * vx[k];
          }
          s = lf_group_sum<TPR>(s);
          dp = lf_group_sum<TPR>(dp);
          if (i >= i1 || mi[u] != 1 || lf_in_window(i, g, P.r, d, P.causal)) continue;
          const float pr = exp2f(s * P.scale_log2 - lse_i[u] * LF_LOG2E);
          const float ds = pr * (dp - dl_i[u]) * P.scale;
#pragma unroll
          for (int k = 0; k < N; k++) {
            ak[k] += ds * q[u][k];
            av[k] += pr * go[u][k];
          }
        }
      }
    }
    // the groups of a warp, then the warps in order
#pragma unroll
    for (int o = TPR; o < 32; o <<= 1)
#pragma unroll
      for (int k = 0; k < N; k++) {
        ak[k] += __shfl_xor_sync(0xffffffffu, ak[k], o);
        av[k] += __shfl_xor_sync(0xffffffffu, av[k], o);
      }
    if (lane < TPR)
#pragma unroll
      for (int k = 0; k < N; k++) {
        s_red[warp][pi * N + k] = ak[k];
        s_red[warp][LF_HD + pi * N + k] = av[k];
      }
    __syncthreads();
    if (warp == 0) {
      float *dst = part + (size_t)un * 2 * LF_HD;
      for (int x = lane; x < 2 * LF_HD; x += 32) {
        float t = 0.f;
        for (int w = 0; w < 8; w++) t += s_red[w][x];
        dst[x] = t;
      }
    }
    __syncthreads();
  }
}

// The same for sequences with several global keys: one block per (b, h,
// group of LF_BW_GCOL_E global keys, chunk of LF_BW_GCOL_ROWS rows), every
// row read once for the group's keys (kept in shared memory, fp32), one
// partial per key in the same fixed order.
#define LF_BW_GCOL_E 4
template <typename T>
__global__ void __launch_bounds__(256, 2)
    lf_bwd_gcol4_kernel(LfDev P, const T *qs, const T *ks, const T *vs, const float *lse,
                        const T *dO, const float *delta, float *part, int nch) {
  constexpr int N = LfVec<T>::N, TPR = LF_HD / N, GPB = 256 / TPR, E = LF_BW_GCOL_E;
  __shared__ float s_red[8][2 * LF_HD];
  __shared__ __align__(16) float s_kv[E][2][LF_HD];  // the group's keys and values
  __shared__ int s_g[E];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int grp = threadIdx.x / TPR, pi = threadIdx.x % TPR;
  const int neg = (P.G + E - 1) / E;
  const long long units = (long long)P.B * P.H * neg * nch;
  for (long long un = blockIdx.x; un < units; un += gridDim.x) {
    const int c = (int)(un % nch);
    const long long be = un / nch;
    const int e0 = (int)(be % neg) * E;
    const long long bh = be / neg;
    const int h = (int)(bh % P.H), b = (int)(bh / P.H), d = P.dil[h], n = P.n;
    const int ng = P.binfo[(size_t)b * LF_BI_WORDS + LF_BI_NG];
    if (e0 >= ng) continue;  // (block-uniform; the reduce reads no partial past ng)
    const int nb = min(E, ng - e0);
    const int32_t *gl = P.gidx + (size_t)b * P.G + e0;
    const size_t base = (size_t)bh * n * LF_HD;
    for (int x = threadIdx.x; x < E * (LF_HD / 2); x += 256) {
      const int e = x / (LF_HD / 2), cc = 2 * (x % (LF_HD / 2));
      float2 kv = make_float2(0.f, 0.f), vv = make_float2(0.f, 0.f);
      if (e < nb) {
        const size_t src = base + (size_t)gl[e] * LF_HD + cc;
        kv = LfIo<T>::ld2(ks + src);
        vv = LfIo<T>::ld2(vs + src);
      }
      s_kv[e][0][cc] = kv.x;
      s_kv[e][0][cc + 1] = kv.y;
      s_kv[e][1][cc] = vv.x;
      s_kv[e][1][cc + 1] = vv.y;
    }
    if (threadIdx.x < E) s_g[threadIdx.x] = (int)threadIdx.x < nb ? gl[threadIdx.x] : -1;
    __syncthreads();
    int gg[E];
#pragma unroll
    for (int e = 0; e < E; e++) gg[e] = s_g[e];
    float ak[E][N], av[E][N];
#pragma unroll
    for (int e = 0; e < E; e++)
#pragma unroll
      for (int k = 0; k < N; k++) ak[e][k] = av[e][k] = 0.f;
    const int32_t *m = P.mask + (size_t)b * n;
    const int i0 = c * LF_BW_GCOL_ROWS, i1 = min(n, i0 + LF_BW_GCOL_ROWS);
    for (int rr = 0; rr < LF_BW_GCOL_ROWS; rr += GPB) {
      // the row's loads all issued together (none waits on a mask test)
      const int i = i0 + rr + grp;
      const int ic = i < i1 ? i : i1 - 1;
      float q[N], go[N];
      LfVec<T>::ld(qs + base + (size_t)ic * LF_HD + pi * N, q);
      LfVec<T>::ld(dO + base + (size_t)ic * LF_HD + pi * N, go);
      const size_t ir = (size_t)bh * n + ic;
      const int mi = m[ic];
      const float lse_i = lse[ir], dl_i = delta[ir];
      const bool row_ok = i < i1 && mi == 1;
#pragma unroll
      for (int e = 0; e < E; e++) {
        float sc = 0.f, dp = 0.f;
#pragma unroll
        for (int k = 0; k < N; k++) {
          sc += q[k] * s_kv[e][0][pi * N + k];
          dp += go[k] * s_kv[e][1][pi * N + k];
        }
        sc = lf_group_sum<TPR>(sc);
        dp = lf_group_sum<TPR>(dp);
        if (!row_ok || gg[e] < 0 || lf_in_window(i, gg[e], P.r, d, P.causal)) continue;
        const float pr = exp2f(sc * P.scale_log2 - lse_i * LF_LOG2E);
        const float ds = pr * (dp - dl_i) * P.scale;
#pragma unroll
        for (int k = 0; k < N; k++) {
          ak[e][k] += ds * q[k];
          av[e][k] += pr * go[k];
        }
      }
    }
    // per key: the groups of a warp, then the warps in order
#pragma unroll
    for (int e = 0; e < E; e++) {
      if (e >= nb) break;  // (block-uniform)
#pragma unroll
      for (int o = TPR; o < 32; o <<= 1)
#pragma unroll
        for (int k = 0; k < N; k++) {
          ak[e][k] += __shfl_xor_sync(0xffffffffu, ak[e][k], o);
          av[e][k] += __shfl_xor_sync(0xffffffffu, av[e][k], o);
        }
      if (lane < TPR)
#pragma unroll
        for (int k = 0; k < N; k++) {
          s_red[warp][pi * N + k] = ak[e][k];
          s_red[warp][LF_HD + pi * N + k] = av[e][k];
        }
      __syncthreads();
      if (warp == 0) {
        float *dst = part + (((size_t)bh * P.G + (e0 + e)) * nch + c) * 2 * LF_HD;
        for (int x = lane; x < 2 * LF_HD; x += 32) {
          float t = 0.f;
          for (int w = 0; w < 8; w++) t += s_red[w][x];
          dst[x] = t;
        }
      }
      __syncthreads();
    }
  }
}

// dK_s[g] += sum of chunks; dV_s[g] likewise.  One block of LF_BW_RED_WARPS
// warps per (b, h, e): warp w sums chunks w, w + LF_BW_RED_WARPS, ... in
// order (four loads in flight), then the warps' sums are added in warp
// order -- a fixed order, so the result is deterministic.
#define LF_BW_RED_WARPS 16
template <typename T>
__global__ void __launch_bounds__(32 * LF_BW_RED_WARPS)
    lf_bwd_gcol_reduce(LfDev P, const float *part, int nch, T *dks, T *dvs) {
  __shared__ float4 s_acc[LF_BW_RED_WARPS][32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // rows (b, h, e) grid-strided; rows past the sequence's global count skip
  for (long long w = blockIdx.x; w < (long long)P.B * P.H * P.G; w += gridDim.x) {
  const int e = (int)(w % P.G);
  const long long bh = w / P.G;
  const int b = (int)(bh / P.H);
  if (e >= P.binfo[(size_t)b * LF_BI_WORDS + LF_BI_NG]) continue;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int c0 = warp; c0 < nch; c0 += 4 * LF_BW_RED_WARPS) {
    float2 a[4], v[4];
#pragma unroll
    for (int u = 0; u < 4; u++) {
      const int c = min(c0 + u * LF_BW_RED_WARPS, nch - 1);
      const float *src = part + ((size_t)w * nch + c) * 2 * LF_HD + 2 * lane;
      a[u] = *reinterpret_cast<const float2 *>(src);
      v[u] = *reinterpret_cast<const float2 *>(src + LF_HD);
    }
#pragma unroll
    for (int u = 0; u < 4; u++) {
      if (c0 + u * LF_BW_RED_WARPS >= nch) break;
      acc.x += a[u].x;
      acc.y += a[u].y;
      acc.z += v[u].x;
      acc.w += v[u].y;
    }
  }
  s_acc[warp][lane] = acc;
  __syncthreads();
  if (warp == 0) {
    float4 t = s_acc[0][lane];
    for (int k = 1; k < LF_BW_RED_WARPS; k++) {
      const float4 x = s_acc[k][lane];
      t.x += x.x;
      t.y += x.y;
      t.z += x.z;
      t.w += x.w;
    }
    const int g = P.gidx[(size_t)b * P.G + e];
    const size_t off = ((size_t)bh * P.n + g) * LF_HD + 2 * lane;
    const float2 kb = LfIo<T>::ld2(dks + off), vb = LfIo<T>::ld2(dvs + off);
    LfIo<T>::st2(dks + off, kb.x + t.x, kb.y + t.y);
    LfIo<T>::st2(dvs + off, vb.x + t.z, vb.y + t.w);
  }
  __syncthreads();  // s_acc is reused by the block's next row
  }
}

// dK_g, dV_g of every key and the dQ_g partials of the global rows in one
// pass over the keys (both need, per key j and global row g, the same
// p_gj = exp(s_gj - lse_g) and dS_gj = p_gj (dP_gj - D_g) scale): one block
// per (b, h, chunk of LF_BW_ROWS_PER_CHUNK keys), grid-strided; a lane group
// (64 / N lanes, 16 bytes each) per key, two keys per group.  Per global
// row the block's dS_gj k_j are added in a fixed order (the groups of a
// warp, then the warps) into the chunk's dQ_g partial, which
// lf_bwd_grow_reduce adds up.  Rows of mask-0 keys are zero.
template <typename T>
__global__ void __launch_bounds__(256)
    lf_bwd_gkey_kernel(LfDev P, const T *qg, const T *kg, const T *vg, const float *lse,
                       const T *dO, const float *delta, T *dkg, T *dvg, float *part_q, int nch) {
  constexpr int N = LfVec<T>::N, TPR = LF_HD / N, GPB = 256 / TPR;
  constexpr int KPG = LF_BW_ROWS_PER_CHUNK / GPB;  // keys per group
  __shared__ float s_red[8][LF_BW_GKEY_EB][LF_HD];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int grp = threadIdx.x / TPR, pi = threadIdx.x % TPR;
  const int n = P.n;
  const long long units = (long long)P.B * P.H * nch;
  for (long long un = blockIdx.x; un < units; un += gridDim.x) {
    const int c = (int)(un % nch);
    const long long bh = un / nch;
    const int b = (int)(bh / P.H);
    const int32_t *m = P.mask + (size_t)b * n;
    const size_t base = (size_t)bh * n * LF_HD + pi * N;
    float kx[KPG][N], vx[KPG][N], ak[KPG][N], av[KPG][N];
    bool on[KPG];
    // the sequence's global count and first global row, read while the keys load
    const int ng = P.binfo[(size_t)b * LF_BI_WORDS + LF_BI_NG];
    const int32_t *gl = P.gidx + (size_t)b * P.G;
    int g_next = P.G > 0 ? gl[0] : 0;  // (the list has G >= 1 entries when G > 0)
#pragma unroll
    for (int kk = 0; kk < KPG; kk++) {
      const int j = c * LF_BW_ROWS_PER_CHUNK + grp + GPB * kk;
      const int jc = min(j, n - 1);
      on[kk] = j < n && m[jc] != 0;
      LfVec<T>::ld(kg + base + (size_t)jc * LF_HD, kx[kk]);
      LfVec<T>::ld(vg + base + (size_t)jc * LF_HD, vx[kk]);
#pragma unroll
      for (int k = 0; k < N; k++) ak[kk][k] = av[kk][k] = 0.f;
    }
    // global rows LF_BW_GKEY_EB at a time: their dQ_g partials are reduced
    // over the block together (two barriers per batch, not per row)
    for (int e0 = 0; e0 < ng; e0 += LF_BW_GKEY_EB) {
      const int nb = min(LF_BW_GKEY_EB, ng - e0);  // (block-uniform)
      float aq[LF_BW_GKEY_EB][N];
#pragma unroll
      for (int u = 0; u < LF_BW_GKEY_EB; u++)
#pragma unroll
        for (int k = 0; k < N; k++) aq[u][k] = 0.f;
#pragma unroll
      for (int u = 0; u < LF_BW_GKEY_EB; u++) {
        if (u >= nb) break;
        const int e = e0 + u;
        const int g = g_next;
        if (e + 1 < ng) g_next = gl[e + 1];
        const size_t gr = (size_t)bh * n + g;
        float q[N], go[N];
        LfVec<T>::ld(qg + base + (size_t)g * LF_HD, q);
        LfVec<T>::ld(dO + base + (size_t)g * LF_HD, go);
        const float L2 = lse[gr] * LF_LOG2E, Dg = delta[gr];
#pragma unroll
        for (int kk = 0; kk < KPG; kk++) {
          float sc = 0.f, dp = 0.f;
#pragma unroll
          for (int k = 0; k < N; k++) {
            sc += q[k] * kx[kk][k];
            dp += go[k] * vx[kk][k];
          }
          sc = lf_group_sum<TPR>(sc);
          dp = lf_group_sum<TPR>(dp);
          if (!on[kk]) continue;
          const float pr = exp2f(sc * P.scale_log2 - L2);
          const float ds = pr * (dp - Dg) * P.scale;
#pragma unroll
          for (int k = 0; k < N; k++) {
            ak[kk][k] += ds * q[k];
            av[kk][k] += pr * go[k];
            aq[u][k] += ds * kx[kk][k];
          }
        }
      }
      // this chunk's dQ_g partials of the batch's rows: the groups of a warp,
      // then the warps in order
#pragma unroll
      for (int u = 0; u < LF_BW_GKEY_EB; u++) {
        if (u >= nb) break;
#pragma unroll
        for (int o = TPR; o < 32; o <<= 1)
#pragma unroll
          for (int k = 0; k < N; k++) aq[u][k] += __shfl_xor_sync(0xffffffffu, aq[u][k], o);
        if (lane < TPR)
#pragma unroll
          for (int k = 0; k < N; k++) s_red[warp][u][pi * N + k] = aq[u][k];
      }
      __syncthreads();
      {
        const int u = threadIdx.x / LF_HD, x = threadIdx.x % LF_HD;
        if (u < nb) {
          float t = 0.f;
          for (int w = 0; w < 8; w++) t += s_red[w][u][x];
          part_q[(((size_t)bh * P.G + (e0 + u)) * nch + c) * LF_HD + x] = t;
        }
      }
      __syncthreads();
    }
#pragma unroll
    for (int kk = 0; kk < KPG; kk++) {
      const int j = c * LF_BW_ROWS_PER_CHUNK + grp + GPB * kk;
      if (j >= n) continue;
      LfVec<T>::st(dkg + base + (size_t)j * LF_HD, ak[kk]);
      LfVec<T>::st(dvg + base + (size_t)j * LF_HD, av[kk]);
    }
  }
}

// dQ_g[g] = sum of chunks: one block per (b, h, e), the order of
// lf_bwd_gcol_reduce.
template <typename T>
__global__ void __launch_bounds__(32 * LF_BW_RED_WARPS)
    lf_bwd_grow_reduce(LfDev P, const float *part, int nch, T *dqg) {
  __shared__ float2 s_acc[LF_BW_RED_WARPS][32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (long long w = blockIdx.x; w < (long long)P.B * P.H * P.G; w += gridDim.x) {
  const int e = (int)(w % P.G);
  const long long bh = w / P.G;
  const int b = (int)(bh / P.H);
  if (e >= P.binfo[(size_t)b * LF_BI_WORDS + LF_BI_NG]) continue;
  float2 acc = make_float2(0.f, 0.f);
  for (int c0 = warp; c0 < nch; c0 += 4 * LF_BW_RED_WARPS) {
    float2 a[4];
#pragma unroll
    for (int u = 0; u < 4; u++) {
      const int c = min(c0 + u * LF_BW_RED_WARPS, nch - 1);
      a[u] = *reinterpret_cast<const float2 *>(part + ((size_t)w * nch + c) * LF_HD + 2 * lane);
    }
#pragma unroll
    for (int u = 0; u < 4; u++) {
      if (c0 + u * LF_BW_RED_WARPS >= nch) break;
      acc.x += a[u].x;
      acc.y += a[u].y;
    }
  }
  s_acc[warp][lane] = acc;
  __syncthreads();
  if (warp == 0) {
    float2 t = s_acc[0][lane];
    for (int k = 1; k < LF_BW_RED_WARPS; k++) {
      t.x += s_acc[k][lane].x;
      t.y += s_acc[k][lane].y;
    }
    const int g = P.gidx[(size_t)b * P.G + e];
    LfIo<T>::st2(dqg + ((size_t)bh * P.n + g) * LF_HD + 2 * lane, t.x, t.y);
  }
  __syncthreads();
  }
}

// ============================================== host

template <typename T>
static cudaError_t lf_bwd_global_parts(const LfLaunch &L, const LfTcBwdArgs &a, const float *delta,
                                       float *part_kv, float *part_q, int nch) {
  const int nchc = (L.dev.n + LF_BW_GCOL_ROWS - 1) / LF_BW_GCOL_ROWS;  // global-column chunks
  const LfDev &D = L.dev;
  cudaError_t e;
  // dQ_g: zero rows outside the global tokens, then the global rows
  e = cudaMemsetAsync(a.dqg, 0, (size_t)D.B * D.H * D.n * LF_HD * sizeof(T), L.stream);
  if (e != cudaSuccess) return e;
  if (D.G > 0) {
    const long long wr = (long long)D.B * D.H * D.G;
    if (D.G >= LF_BW_GCOL_E) {  // several global keys: each row read once per group of keys
      const long long wk = (long long)D.B * D.H * ((D.G + LF_BW_GCOL_E - 1) / LF_BW_GCOL_E) * nchc;
      const unsigned ugrid = (unsigned)std::min<long long>(wk, 148LL * 16);  // grid-strided units
      lf_bwd_gcol4_kernel<T><<<ugrid, 256, 0, L.stream>>>(
          D, (const T *)a.qs, (const T *)a.ks, (const T *)a.vs, a.lse, (const T *)a.dO, delta, part_kv, nchc);
    } else {
      const long long wk = (long long)D.B * D.H * D.G * nchc;
      const unsigned ugrid = (unsigned)std::min<long long>(wk, 148LL * 16);  // grid-strided units
      lf_bwd_gcol_kernel<T><<<ugrid, 256, 0, L.stream>>>(
          D, (const T *)a.qs, (const T *)a.ks, (const T *)a.vs, a.lse, (const T *)a.dO, delta, part_kv, nchc);
    }
    const unsigned rgrid = (unsigned)std::min<long long>(wr, 4096);
    lf_bwd_gcol_reduce<T><<<rgrid, 32 * LF_BW_RED_WARPS, 0, L.stream>>>(D, part_kv, nchc, (T *)a.dks,
                                                                        (T *)a.dvs);
    lf_bwd_grow_reduce<T><<<rgrid, 32 * LF_BW_RED_WARPS, 0, L.stream>>>(D, part_q, nch, (T *)a.dqg);
    lf_launches_add(3);
  }
  return cudaGetLastError();
}

cudaError_t lf_launch_bwd_delta(const LfLaunch &L, const void *o, const void *dO, float *delta);

int lf_tc_bwd(const LfLaunch &L, const LfTcBwdArgs &a, char *err, size_t errlen) {
  const LfDev &D = L.dev;
  const int f16 = L.dtype == LF_F16 ? 1 : 0;
  float *delta = (float *)(L.ws_base + L.ws.delta);
  cudaError_t ce;
  // delta = rowsum(dO * O); then dK_g, dV_g of every key and the dQ_g
  // partials, in one pass over the keys
  const int nch = (D.n + LF_BW_ROWS_PER_CHUNK - 1) / LF_BW_ROWS_PER_CHUNK;
  float *part_kv = (float *)(L.ws_base + L.ws.part_acc), *part_q = (float *)(L.ws_base + L.ws.part_ml);
  ce = lf_launch_bwd_delta(L, a.o, a.dO, delta);
  if (ce == cudaSuccess) {
    const unsigned kgrid = (unsigned)std::min<long long>((long long)D.B * D.H * nch, 148LL * 16);
    if (f16)
      lf_bwd_gkey_kernel<__half><<<kgrid, 256, 0, L.stream>>>(
          D, (const __half *)a.qg, (const __half *)a.kg, (const __half *)a.vg, a.lse,
          (const __half *)a.dO, delta, (__half *)a.dkg, (__half *)a.dvg, part_q, nch);
    else
      lf_bwd_gkey_kernel<__nv_bfloat16><<<kgrid, 256, 0, L.stream>>>(
          D, (const __nv_bfloat16 *)a.qg, (const __nv_bfloat16 *)a.kg, (const __nv_bfloat16 *)a.vg,
          a.lse, (const __nv_bfloat16 *)a.dO, delta, (__nv_bfloat16 *)a.dkg, (__nv_bfloat16 *)a.dvg,
          part_q, nch);
    lf_launches_add(1);
    ce = cudaGetLastError();
  }
  if (ce != cudaSuccess) {
    snprintf(err, errlen, "backward delta / dK_g launch: %s", cudaGetErrorString(ce));
    return LF_ERR_CUDA;
  }
  LfBwParams P;
  memset(&P, 0, sizeof(P));
  P.dev = D;
  const uint64_t n = D.n, H = D.H, B = D.B, rowb = 128;
  int nmaps = 0, nseg = 0, start = 0;
  std::map<std::pair<int, int>, int> rmap;
  for (int h0 = 0; h0 < D.H;) {
    int h1 = h0 + 1;
    while (h1 < D.H && D.dil[h1] == D.dil[h0]) h1++;
    const int d = D.dil[h0];
    for (int rho = 0; rho < d; rho++) {
      const int cnt = lf_sub_len(D.n, d, rho);
      const int nqb = (cnt + LF_BQ - 1) / LF_BQ;
      if (nqb == 0) continue;
      auto key = std::make_pair(d, rho);
      if (!rmap.count(key)) {
        if (nmaps + 8 > LF_BW_MAX_MAPS - 2) {
          snprintf(err, errlen,
                   "tensor-core backward: too many distinct dilation residues (the sum of the "
                   "distinct dilations must stay <= %d)", (LF_BW_MAX_MAPS - 2) / 8);
          return LF_ERR_UNSUPPORTED;
        }
        const char *srcs[4] = {(const char *)a.qs, (const char *)a.ks, (const char *)a.vs,
                               (const char *)a.dO};
        for (int k = 0; k < 8; k++)
          if (!lf_make_map(&P.maps[nmaps + k], f16, srcs[k & 3] + rho * rowb, cnt, H, B, d * rowb,
                           n * rowb, H * n * rowb, k < 4 ? LF_BQ : LF_BW_BK)) {
            snprintf(err, errlen, "tensor map encode failed (backward, d=%d, rho=%d)", d, rho);
            return LF_ERR_CUDA;
          }
        rmap[key] = nmaps;
        nmaps += 8;
      }
      if (nseg >= LF_BW_MAX_SEG) {
        snprintf(err, errlen, "tensor-core backward: too many head/residue segments");
        return LF_ERR_UNSUPPORTED;
      }
      P.seg[nseg] = LfTcSeg{h0, h1, d, rho, cnt, nqb, start, rmap[key]};
      start += (h1 - h0) * nqb;
      nseg++;
    }
    h0 = h1;
  }
  P.nseg = nseg;
  P.per_batch = start;
  const int Ga = L.ws.G, Gka = L.ws.Gk;
  char *qg_c = L.ws_base + L.ws.qg_c, *ks_c = L.ws_base + L.ws.ks_c, *vs_c = L.ws_base + L.ws.vs_c;
  P.gbox = std::min(Gka, LF_BW_BK);
  P.map_ksc = nmaps;
  P.map_vsc = nmaps + 1;
  if (!lf_make_map(&P.maps[nmaps], f16, ks_c, Gka, H, B, rowb, Gka * rowb, H * Gka * rowb, P.gbox) ||
      !lf_make_map(&P.maps[nmaps + 1], f16, vs_c, Gka, H, B, rowb, Gka * rowb, H * Gka * rowb, P.gbox)) {
    snprintf(err, errlen, "tensor map encode failed (backward global maps)");
    return LF_ERR_CUDA;
  }
  P.lse = a.lse;
  P.delta = delta;
  if (D.G > 0) {
    ce = lf_launch_gather(L, a.qg, a.ks, a.vs, qg_c, ks_c, vs_c, Ga, Gka);
    if (ce != cudaSuccess) {
      snprintf(err, errlen, "gather launch: %s", cudaGetErrorString(ce));
      return LF_ERR_CUDA;
    }
  }
  // one launch: dK/dV blocks (rows = keys), then dQ blocks (rows = queries)
  const unsigned grid = (unsigned)(2LL * D.B * P.per_batch);
  {
    void (*kern)(const LfBwParams) = f16 ? lf_tc_bwd_kernel<1> : lf_tc_bwd_kernel<0>;
    ce = lf_kernel_smem((const void *)kern, LF_BW_SMEM);
    if (ce != cudaSuccess) {
      snprintf(err, errlen, "cudaFuncSetAttribute (backward): %s", cudaGetErrorString(ce));
      return LF_ERR_CUDA;
    }
    P.dq_out = a.dqs;
    P.dk_out = a.dks;
    P.dv_out = a.dvs;
    kern<<<grid, LF_BW_THREADS, LF_BW_SMEM, L.stream>>>(P);
    lf_launches_add(1);
    ce = cudaGetLastError();
    if (ce != cudaSuccess) {
      snprintf(err, errlen, "tensor-core backward launch: %s", cudaGetErrorString(ce));
      return LF_ERR_CUDA;
    }
  }
  // global-column part of dK_s / dV_s (after the band part) and dQ_g
  ce = f16 ? lf_bwd_global_parts<__half>(L, a, delta, part_kv, part_q, nch)
           : lf_bwd_global_parts<__nv_bfloat16>(L, a, delta, part_kv, part_q, nch);
  if (ce != cudaSuccess) {
    snprintf(err, errlen, "backward global parts: %s", cudaGetErrorString(ce));
    return LF_ERR_CUDA;
  }
  return LF_OK;
}

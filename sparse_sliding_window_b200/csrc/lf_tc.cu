// lf_tc.cu -- tensor-core (tcgen05 / TMEM / TMA) forward of Longformer
// attention for sm_100a, bf16 or f16 inputs, fp32 accumulation.
//
// One kernel runs two kinds of work items:
//
//  * BAND items: 128 query rows t0..t0+127 of one (b, h, residue rho).  A
//    head with dilation d is split into its d residue sub-sequences
//    rho, rho+d, ... ("gaps of size d": segmentfault page, section
//    扩张滑动窗口); in sub-sequence coordinates the window is a plain band of
//    radius r (causal: [t-r, t]), so the CTA walks only the key tiles that
//    intersect the band (page section 实现: only a fixed number of diagonals
//    of QK^T are computed).  The residue view is a TMA tensor map whose row
//    stride is d rows, so dilated heads need no gather.  After the band tiles
//    come the global-column tiles: the K_s/V_s rows of the sequence's global
//    tokens (compacted by lf_gather_kernel), minus the keys already inside
//    the row's window (the union of the glossary example), merged into the
//    same online softmax.  Global query rows are skipped (their output comes
//    from the global-row items); mask-0 rows get o = 0, lse = -inf.
//  * GLOBAL items: up to 128 global query rows (Q_g, compacted) against a
//    chunk of LF_TC_CHUNK_TILES key tiles of K_g / V_g (every valid key:
//    global attention sees the whole sequence, segmentfault page section
//    全局注意力).  Each writes an unnormalised partial (acc, max, sum) that
//    lf_combine_kernel merges (split-KV).
//
// Persistent: one CTA of 384 threads per SM runs two independent streams.
// Stream g has its own producer warp (8 + 2g: takes the next work item and
// issues its TMA loads -- Q into the stream's buffer, K/V tiles into its
// 3-stage ring), MMA warp (9 + 2g: issues the tcgen05.mma phases from one
// elected lane), four softmax warps (4g .. 4g+3: one TMEM lane = one query
// row per thread) and 256 TMEM columns (S tile, O accumulator, P tile).  A
// stream processes whole items, so nothing is merged between streams; while
// one stream waits for its next S tile the other keeps the SM's exp unit
// busy.  Items come largest first, from the CTA's own list when there are
// few per SM and from one grid-wide counter otherwise.
// Per tile t of an item:
//             SMX  attend mask of the row for tile t (while S is in flight)
//             MMA  S = Q K_t^T                            -> commit s_full
//             SMX  P = exp2(S*scale*log2e - m) against the row's running
//                  reference m (the tile is redone with its own max, O
//                  rescaled, when the row sum leaves the P format's safe
//                  range), row sum                       -> arrive p_full
//             MMA  S = Q K_{t+1}^T                        -> commit s_full
//             MMA  O += P V_t (A operand from TMEM)       -> kv_empty, pv_done
// After the item's last tile the softmax warps write O / l and the
// log-normaliser, so the n x w score band never leaves the SM.
//
// Every wait is bounded: after LF_WAIT_NS without progress the waiting
// thread records LF_ERR_DEVICE_TIMEOUT in the status word, raises the CTA's
// abort flag and leaves its loop; all roles meet at the final barrier and
// the TMEM columns are freed before the CTA exits.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <map>
#include <utility>
#include <vector>

#include "lf_ptx.cuh"
#include "lf_tc.cuh"

#define LF_TC_THREADS 384
#define LF_TC_NS 3
#define LF_TC_MAX_MAPS 192  // kernel parameters may take up to 32 KB
#define LF_TC_MAX_SEG 96

// TMEM column map: stream g owns columns [256g, 256g + 256): its S tile,
// O accumulator and P tile (bf16/f16 pairs, the A operand of P.V)
#define LF_TM_S(g) ((g)*256)
#define LF_TM_O(g) ((g)*256 + 128)
#define LF_TM_P(g) ((g)*256 + 192)
#define LF_TM_COLS 512

// shared memory map (bytes from the 1024-aligned base): per stream a Q
// buffer and LF_TC_NS stages of (K tile, V tile); then the barriers, the
// TMEM slot, the abort flag and the work-item slots
#define LF_SM_STREAM (16384 + LF_TC_NS * 32768)
#define LF_SM_Q(g) ((g)*LF_SM_STREAM)
#define LF_SM_K(g, s) ((g)*LF_SM_STREAM + 16384 + (s)*32768)
#define LF_SM_V(g, s) ((g)*LF_SM_STREAM + 16384 + (s)*32768 + 16384)
#define LF_SM_BAR (2 * LF_SM_STREAM)
#define LF_SMEM_BYTES (LF_SM_BAR + 1024)
static_assert(96 + 16 * LF_TC_NS <= 160, "per-stream barrier block");
static_assert(LF_SMEM_BYTES <= 232448, "shared memory per CTA");


struct LfTcParams {
  CUtensorMap maps[LF_TC_MAX_MAPS];
  LfDev dev;
  LfTcSeg seg[LF_TC_MAX_SEG];
  int nseg, per_batch, n_gitems, ngq, gbox;
  int sched_cta;  // 1: per-CTA item lists, 0: one grid-wide item counter
  int map_kg, map_vg, map_qgc, map_ksc, map_vsc;
  int f16;
  void *o;
  float *lse;
  float *part_acc;
  float2 *part_ml;
};


// P for one S tile of this thread's TMEM lane against the reference m:
// p = 2^(s*sl2 - m) for the attended columns (bit set in w), 0 elsewhere,
// packed into P, summed into lt; with want_max the attended max of the raw
// scores goes to mx instead and nothing is written.  TMEM loads run one
// 32-column chunk ahead of the arithmetic; the arithmetic of chunks no lane
// of the warp attends is skipped (P written as zeros).
template <int kF16>
__device__ __forceinline__ void lf_tile_pass(uint32_t tS, uint32_t tP, const uint32_t (&w)[4],
                                             float sl2, float m, float &lt, float &mx,
                                             bool want_max, LfPvGate &gate) {
  bool anyc[4];
#pragma unroll
  for (int cc = 0; cc < 4; cc++) anyc[cc] = __any_sync(0xffffffffu, w[cc] != 0u);
  const float mneg = -m;
  uint32_t buf[2][32];  // chunk cc lives in buf[cc & 1]; chunk cc+1 loads while cc computes
  float s0 = 0.f, s1 = 0.f, m0 = -INFINITY, m1 = -INFINITY;
  lf_tmem_ld32_nowait(tS, buf[0]);
#pragma unroll
  for (int cc = 0; cc < 4; cc++) {
    uint32_t(&x)[32] = buf[cc & 1];
    lf_tmem_wait_ld_regs(x);
    if (cc + 1 < 4) lf_tmem_ld32_nowait(tS + 32 * (cc + 1), buf[(cc + 1) & 1]);
    if (!anyc[cc]) {
      if (!want_max) {
        gate.pass();
        uint32_t z[16];
#pragma unroll
        for (int k = 0; k < 16; k++) z[k] = 0u;
        lf_tmem_st16(tP + 16 * cc, z);
      }
      continue;
    }
    const uint32_t wc = w[cc];
    if (!__all_sync(0xffffffffu, wc == 0xffffffffu)) {
#pragma unroll
      for (int k = 0; k < 32; k++) x[k] = ((wc >> k) & 1u) ? x[k] : 0xff800000u;  // -inf
    }
    if (want_max) {
#pragma unroll
      for (int k = 0; k < 32; k += 2) {
        m0 = fmaxf(m0, __uint_as_float(x[k]));
        m1 = fmaxf(m1, __uint_as_float(x[k + 1]));
      }
    } else {
      uint32_t pw[16];
#pragma unroll
      for (int k = 0; k < 32; k += 2) {
        const float p0 = lf_ex2(fmaf(__uint_as_float(x[k]), sl2, mneg));
        const float p1 = lf_ex2(fmaf(__uint_as_float(x[k + 1]), sl2, mneg));
        s0 += p0;
        s1 += p1;
        pw[k / 2] = lf_pack2<kF16>(p0, p1);
      }
      gate.pass();
      lf_tmem_st16(tP + 16 * cc, pw);
    }
  }
  if (want_max) mx = fmaxf(m0, m1);
  else lt = s0 + s1;
}

// A decoded work item (every role decodes the same sequence).
struct LfItem {
  int gitem, b, h, d, rho, cnt, qrow0, mq, mk, mv, nband, nglob, T, kt0, ng;
};

__device__ __forceinline__ bool lf_decode(const LfTcParams &P, int idx, LfItem &it) {
  const LfDev &D = P.dev;
  const int n = D.n;
  it.d = 1;
  it.rho = 0;
  it.cnt = n;
  it.kt0 = 0;
  it.nglob = 0;
  if (idx < P.n_gitems) {
    it.gitem = 1;
    const int c = idx % D.nch;
    idx /= D.nch;
    const int qt = idx % P.ngq;
    idx /= P.ngq;
    it.h = idx % D.H;
    it.b = idx / D.H;
    it.ng = D.binfo[(size_t)it.b * LF_BI_WORDS + LF_BI_NG];
    it.qrow0 = qt * LF_BQ;
    it.kt0 = c * D.chunk_tiles;
    const int ktiles = (n + LF_BK - 1) / LF_BK;
    it.nband = min(D.chunk_tiles, ktiles - it.kt0);
    it.mq = P.map_qgc;
    it.mk = P.map_kg;
    it.mv = P.map_vg;
    it.T = it.nband;
    return it.qrow0 < it.ng && it.nband > 0;  // false: nothing to do
  }
  it.gitem = 0;
  idx -= P.n_gitems;
  it.b = idx / P.per_batch;
  int rem = idx - it.b * P.per_batch;
  int s = 0;
  while (s + 1 < P.nseg && rem >= P.seg[s + 1].start) s++;
  const LfTcSeg &sg = P.seg[s];
  rem -= sg.start;
  it.h = sg.h0 + rem / sg.nqb;
  it.qrow0 = (rem % sg.nqb) * LF_BQ;
  it.d = sg.d;
  it.rho = sg.rho;
  it.cnt = sg.cnt;
  it.mq = sg.map;
  it.mk = sg.map + 1;
  it.mv = sg.map + 2;
  it.nband = lf_band_tiles(D.r, D.causal);
  const int32_t *bi = D.binfo + (size_t)it.b * LF_BI_WORDS;
  it.ng = bi[LF_BI_NG];
  bool need = it.ng > 0;
  if (need && it.d == 1 && !D.causal) {
    // every global key inside every row's window: the band covers them
    const int tlast = min(it.qrow0 + LF_BQ - 1, it.cnt - 1);
    if (bi[LF_BI_GMIN] >= tlast - D.r && bi[LF_BI_GMAX] <= it.qrow0 + D.r) need = false;
  }
  it.nglob = need ? (it.ng + LF_BK - 1) / LF_BK : 0;
  it.T = it.nband + it.nglob;
  return true;
}

// ------------------------------------------------------------ the kernel

template <int kF16>
__global__ void __launch_bounds__(LF_TC_THREADS, 1)
    lf_tc_fwd_kernel(const __grid_constant__ LfTcParams P) {
  extern __shared__ __align__(1024) uint8_t lf_smem_raw[];
  // the dynamic shared window starts 1024-byte aligned (128-byte swizzled
  // TMA tiles need it); checked rather than padded
  const uint32_t sbase = lf_smem(lf_smem_raw);
  uint8_t *gbase = lf_smem_raw;
  if (sbase & 1023u) {
    if (threadIdx.x == 0) lf_set_status(P.dev.status, LF_ERR_UNSUPPORTED, 9000);
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const LfDev &D = P.dev;
  const int n = D.n;
  const int nitems = P.n_gitems + D.B * P.per_batch;
  // stream of this warp: softmax warps 0-3 / 4-7, producer 8 / 10, MMA 9 / 11
  const int g = warp < 8 ? warp >> 2 : (warp - 8) >> 1;

  // barriers of stream g (8 bytes each, 12 + 2 LF_TC_NS per stream, 160-byte stride)
  const uint32_t bar = sbase + LF_SM_BAR + 160 * g;
  const uint32_t q_full = bar, q_empty = bar + 8, s_full = bar + 16, p_full = bar + 24,
                 pv_done = bar + 32, o_full = bar + 40, o_free = bar + 48, end_bar = bar + 56;
  const uint32_t it_full0 = bar + 64, it_empty0 = bar + 80, kv_full0 = bar + 96,
                 kv_empty0 = bar + 96 + 8 * LF_TC_NS;
  uint32_t *tmem_slot = (uint32_t *)(gbase + LF_SM_BAR + 512);
  volatile int *item_slot = (volatile int *)(gbase + LF_SM_BAR + 520) + 2 * g;  // [2] per stream
  volatile int *abort_flag = (volatile int *)(gbase + LF_SM_BAR + 536);  // [2]: flag, wait limit
  int *cta_next = (int *)(gbase + LF_SM_BAR + 544);  // the CTA's next work item, shared by its streams

  if (threadIdx.x == 0) {
    for (int gg = 0; gg < 2; gg++) {
      const uint32_t b0 = sbase + LF_SM_BAR + 160 * gg;
      lf_mbar_init(b0, 1);       // q_full
      lf_mbar_init(b0 + 8, 1);   // q_empty
      lf_mbar_init(b0 + 16, 1);  // s_full
      lf_mbar_init(b0 + 24, 4);  // p_full (four softmax warps)
      lf_mbar_init(b0 + 32, 1);  // pv_done
      lf_mbar_init(b0 + 40, 1);  // o_full
      lf_mbar_init(b0 + 48, 4);  // o_free (four softmax warps)
      lf_mbar_init(b0 + 56, 1);  // end
      for (int i = 0; i < 2; i++) {
        lf_mbar_init(b0 + 64 + 8 * i, 1);  // item slot filled
        lf_mbar_init(b0 + 80 + 8 * i, 5);  // item slot read (MMA warp + four softmax warps)
      }
      for (int s = 0; s < LF_TC_NS; s++) {
        lf_mbar_init(b0 + 96 + 8 * s, 1);
        lf_mbar_init(b0 + 96 + 8 * LF_TC_NS + 8 * s, 1);
      }
    }
    abort_flag[0] = 0;
    abort_flag[1] = P.dev.wait_us;
    *cta_next = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 9) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     lf_smem(tmem_slot)),
                 "r"(LF_TM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  lf_tc_fence_before();
  __syncthreads();
  lf_tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // launched as a programmatic dependent of the mask pass: the set-up above
  // overlaps its tail; its tables (global list, ranks, compacted rows) are
  // read only after it has completed
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");  // the combine kernel

  // consumers take the stream's items from its two slots in order; -1 ends
  auto take_item = [&](int k, int &idx) -> bool {
    const int slot = k & 1;
    if (!lf_wait_warp(it_full0 + 8 * slot, (k >> 1) & 1, abort_flag, D.status, 15)) return false;
    idx = item_slot[slot];
    __syncwarp();
    if (lane == 0) lf_mbar_arrive(it_empty0 + 8 * slot);
    return true;
  };

  if (warp == 8 || warp == 10) {
    // ================================================== TMA producer + scheduler
    if (lane == 0) {
      int gt = 0, k = 0, qk = -1;
      bool ok = true;
      // test hook: each stream of CTA 0 leaves one K/V stage (its tile
      // skip_tile - 1) unloaded, so the MMA warp's bounded wait for it
      // expires (LF_ERR_DEVICE_TIMEOUT) and the CTA aborts
      const int skip = (D.skip_tile > 0 && blockIdx.x == 0) ? D.skip_tile - 1 : -1;
      while (ok) {
        // next work item (largest first: global rows, then band blocks);
        // empty items are skipped.  With many items per CTA they come from
        // one grid-wide counter (balance over the whole grid); with a few,
        // each CTA walks its own list blockIdx.x, blockIdx.x + gridDim.x, ...,
        // taken by whichever of its two streams is free -- so a CTA's last
        // item mostly runs alone instead of two late items sharing an SM.
        int idx;
        LfItem it;
        for (;;) {
          idx = P.sched_cta ? blockIdx.x + gridDim.x * atomicAdd(cta_next, 1)
                            : atomicAdd(D.status + LF_ST_SCHED, 1);
          if (idx >= nitems) {
            idx = -1;
            break;
          }
          if (lf_decode(P, idx, it)) break;
        }
        const int slot = k & 1;
        if (k >= 2 &&
            !lf_wait_fast(it_empty0 + 8 * slot, ((k >> 1) & 1) ^ 1, abort_flag, D.status, 16)) {
          ok = false;
          break;
        }
        item_slot[slot] = idx;
        lf_mbar_arrive(it_full0 + 8 * slot);
        if (idx < 0) break;
        // the previous item's scores all computed: Q may be replaced
        if (k >= 1 && !lf_wait_fast(q_empty, (k - 1) & 1, abort_flag, D.status, 1)) {
          ok = false;
          break;
        }
        lf_mbar_expect_tx(q_full, 16384);
        lf_tma_load4(sbase + LF_SM_Q(g), &P.maps[it.mq], q_full, 0, it.qrow0, it.h, it.b);
        qk = k;
        const int tk0 = it.qrow0 - D.r;
        for (int t = 0; t < it.T; t++, gt++) {
          const int s = gt % LF_TC_NS;
          if (gt >= LF_TC_NS &&
              !lf_wait_fast(kv_empty0 + 8 * s, ((gt / LF_TC_NS) & 1) ^ 1, abort_flag, D.status, 2)) {
            ok = false;
            break;
          }
          if (gt == skip) continue;
          int row;
          const CUtensorMap *km, *vm;
          uint32_t bytes;
          if (t < it.nband) {
            row = it.gitem ? (it.kt0 + t) * LF_BK : tk0 + t * LF_BK;
            km = &P.maps[it.mk];
            vm = &P.maps[it.mv];
            bytes = 2 * 16384;
          } else {
            row = (t - it.nband) * LF_BK;
            km = &P.maps[P.map_ksc];
            vm = &P.maps[P.map_vsc];
            bytes = 2 * P.gbox * 128;
          }
          lf_mbar_expect_tx(kv_full0 + 8 * s, bytes);
          lf_tma_load4(sbase + LF_SM_K(g, s), km, kv_full0 + 8 * s, 0, row, it.h, it.b);
          lf_tma_load4(sbase + LF_SM_V(g, s), vm, kv_full0 + 8 * s, 0, row, it.h, it.b);
        }
        k++;
      }
      if (*abort_flag) {
        // let the copies already issued land before the CTA exits
        for (int i = max(0, gt - LF_TC_NS); i < gt; i++)
          if (i != skip) lf_wait_drain(kv_full0 + 8 * (i % LF_TC_NS), (i / LF_TC_NS) & 1, D.status, 11);
        if (qk >= 0) lf_wait_drain(q_full, qk & 1, D.status, 13);
      }
    }
  } else if (warp == 9 || warp == 11) {
    // ================================================== MMA issuer
    // The whole warp waits; one elected lane issues each phase.  Per tile t
    // of an item: wait P(t), issue S(t + 1) (S is free once P(t) is
    // written), then O (+)= P(t) V_t.
    const uint64_t dq0 = lf_sdesc(sbase + LF_SM_Q(g), 16, 1024);
    const uint64_t dk0 = lf_sdesc(sbase + LF_SM_K(g, 0), 16, 1024);
    const uint64_t dv0 = lf_sdesc(sbase + LF_SM_V(g, 0), 0, 1024);
    const uint32_t id_pv = lf_idesc(kF16, 64, 1);
    int gt = 0, k = 0;
    bool ok = true;
    while (ok) {
      int idx;
      if (!take_item(k, idx)) {
        ok = false;
        break;
      }
      if (idx < 0) break;
      LfItem it;
      lf_decode(P, idx, it);
      const int ngk = (it.ng + 15) / 16 * 16;  // global key tile width, multiple of 16
      auto ncols = [&](int t) { return t < it.nband ? LF_BK : min(LF_BK, ngk - (t - it.nband) * LF_BK); };
      auto issue_s = [&](int t) -> bool {
        const int j = gt + t, s = j % LF_TC_NS;
        if (!lf_wait_warp(kv_full0 + 8 * s, (j / LF_TC_NS) & 1, abort_flag, D.status, 4)) return false;
        lf_tc_fence_after();
        lf_mma_s_phase(tmem + LF_TM_S(g), dq0, dk0 + (uint64_t)(s * (32768 >> 4)),
                       lf_idesc(kF16, ncols(t), 0), s_full);
        if (t + 1 == it.T) lf_commit_w(q_empty);  // every S of the item issued
        return true;
      };
      if (!lf_wait_warp(q_full, k & 1, abort_flag, D.status, 3)) {
        ok = false;
        break;
      }
      if (!issue_s(0)) {
        ok = false;
        break;
      }
      for (int t = 0; t < it.T && ok; t++) {
        const int j = gt + t;
        // P(t) written and S(t) consumed by the softmax warps
        if (!lf_wait_warp(p_full, j & 1, abort_flag, D.status, 5)) {
          ok = false;
          break;
        }
        lf_tc_fence_after();
        if (t + 1 < it.T && !issue_s(t + 1)) {
          ok = false;
          break;
        }
        // O read out by the softmax warps at the end of the previous item
        if (t == 0 && k >= 1 && !lf_wait_warp(o_free, (k - 1) & 1, abort_flag, D.status, 6)) {
          ok = false;
          break;
        }
        const int s = j % LF_TC_NS;
        lf_mma_ts_phase(tmem + LF_TM_O(g), tmem + LF_TM_P(g), dv0 + (uint64_t)(s * (32768 >> 4)),
                        2048 >> 4, id_pv, (1u << (ncols(t) / 16)) - 1u, t > 0 ? 1u : 0u,
                        kv_empty0 + 8 * s, pv_done, t + 1 == it.T ? o_full : 0u);
      }
      k++;
      gt += it.T;
    }
    // every MMA this warp issued has completed once end_bar flips (also
    // after an abort: TMEM is freed after this)
    lf_commit_w(end_bar);
    lf_wait_drain(end_bar, 0, D.status, 7);
    __syncwarp();
  } else if (warp < 8) {
    // ================================================== softmax warps
    // warps 4g .. 4g+3 of stream g: one TMEM lane = one query row per thread
    const int quarter = warp & 3;
    const int q = quarter * 32 + lane;  // query row of the tile == TMEM lane
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_off + LF_TM_S(g), tP = tmem + lane_off + LF_TM_P(g);
    const uint32_t tO = tmem + lane_off + LF_TM_O(g);
    const float sl2 = D.scale_log2;
    // loop-invariant parameters held in registers (not re-read from the
    // parameter bank inside the tile loop)
    const int rr = lf_reg(D.r), causal = lf_reg(D.causal);
    // per-row context of a work item: taken, decoded and its global loads
    // issued before the previous item's epilogue, which hides their latency
    struct Ctx {
      LfItem it;
      int code, pos, e_lo, e_hi;
      bool active, padded;
    };
    auto setup = [&](int kk, Ctx &c) -> int {  // 1: item, 0: no more items, -1: aborted
      int idx;
      if (!take_item(kk, idx)) return -1;
      if (idx < 0) return 0;
      lf_decode(P, idx, c.it);
      const int32_t *mr = D.mask + (size_t)c.it.b * n;
      c.code = 0;
      c.pos = 0;
      if (c.it.gitem) {
        c.active = c.it.qrow0 + q < c.it.ng;
      } else {
        const int t = c.it.qrow0 + q;
        if (t < c.it.cnt) {
          c.pos = c.it.rho + t * c.it.d;
          c.code = mr[c.pos];
        }
        c.active = (c.code == 1);
      }
      c.padded = D.binfo[(size_t)c.it.b * LF_BI_WORDS + LF_BI_NVALID] < n;
      // global keys already in the row's window: index range [e_lo, e_hi) of
      // the sorted global list, from the rank array (filtered by residue)
      c.e_lo = 0;
      c.e_hi = 0;
      if (!c.it.gitem && c.it.nglob > 0 && c.active) {
        const int32_t *gr = D.grank + (size_t)c.it.b * (n + 1);
        c.e_lo = gr[max(c.pos - rr * c.it.d, 0)];
        c.e_hi = gr[min((causal ? c.pos : c.pos + rr * c.it.d) + 1, n)];
      }
      return 1;
    };
    int gt = 0, k = 0;
    bool alive = true;
    Ctx cur;
    int st = setup(0, cur);
    alive = st >= 0;
    while (st == 1) {
      const LfItem &it = cur.it;
      const int code = cur.code, pos = cur.pos, e_lo = cur.e_lo, e_hi = cur.e_hi;
      const bool active = cur.active, padded = cur.padded;
      const int32_t *mrow = D.mask + (size_t)it.b * n;
      const int32_t *gl = D.gidx + (size_t)it.b * D.G;
      const int tk0 = it.qrow0 - rr;
      float m_ref = 0.f, l = 0.f;
      for (int t = 0; t < it.T; t++) {
        const int j = gt + t;
        // ---- attend mask of row q over the tile's 128 columns (4 words);
        // computed while the tile's scores are still on their way
        uint32_t w[4];
        if (t < it.nband) {
          const int kb = it.gitem ? (it.kt0 + t) * LF_BK : tk0 + t * LF_BK;
          int lo = 0, hi = LF_BK - 1;
          if (!it.gitem) lf_band_cols(q, t, rr, causal, lo, hi);
          lo = max(lo, -kb);  // keys exist on [0, cnt)
          hi = min(hi, it.cnt - 1 - kb);
          if (!active) hi = -1;
#pragma unroll
          for (int cc = 0; cc < 4; cc++) w[cc] = lf_range_bits(lo, hi, 32 * cc);
          if (padded) {
#pragma unroll
            for (int cc = 0; cc < 4; cc++) {
              const int tk = kb + 32 * cc + lane;
              const bool okk = tk >= 0 && tk < it.cnt && mrow[it.rho + tk * it.d] != 0;
              w[cc] &= __ballot_sync(0xffffffffu, okk);
            }
          }
        } else {
          const int gbs = (t - it.nband) * LF_BK;
          const int hi = active ? min(LF_BK - 1, it.ng - 1 - gbs) : -1;
#pragma unroll
          for (int cc = 0; cc < 4; cc++) {
            uint32_t inwin = lf_range_bits(e_lo - gbs, e_hi - 1 - gbs, 32 * cc);
            if (it.d > 1) {
              const int e = gbs + 32 * cc + lane;
              const bool res = e < it.ng && (gl[e] - it.rho) % it.d == 0;
              inwin &= __ballot_sync(0xffffffffu, res);
            }
            w[cc] = lf_range_bits(0, hi, 32 * cc) & ~inwin;
          }
        }
        if (!lf_wait_warp(s_full, j & 1, abort_flag, D.status, 8)) {
          alive = false;
          break;
        }
        lf_tc_fence_after();
        // ---- probabilities of the tile -> P (TMEM) against the running
        // reference m_ref (0 until a tile says otherwise).  The tile's row sum
        // shows when the reference is off: a sum above 2^15 means some p may
        // exceed the P format (f16) -- the row max grew; a sum below kLowT on
        // a row whose running sum is also below kLowL means the tile's
        // largest p have left the P format's precise range (f16 normals end
        // at 2^-14, the ex2 flush at 2^-126) while they still matter to the
        // row.  Either way the warp redoes the tile with the tile's own max
        // (O rescaled).  P(t - 1) must have been consumed before P is written.
        LfPvGate gate{pv_done, j > 0 ? (j - 1) & 1 : -1, abort_flag, D.status};
        const bool any_bits = (w[0] | w[1] | w[2] | w[3]) != 0u;
        float lt = 0.f, mx = -INFINITY;
        lf_tile_pass<kF16>(tS, tP, w, sl2, m_ref, lt, mx, false, gate);
        constexpr float kLowT = kF16 ? 0.0625f : 9.3e-10f, kLowL = kF16 ? 1.f : 9.3e-10f;
        const bool off = any_bits && (lt > 32768.f || (lt < kLowT && l < kLowL));
        if (__any_sync(0xffffffffu, off)) {
          lf_tile_pass<kF16>(tS, tP, w, sl2, m_ref, lt, mx, true, gate);  // max only
          const float ms = mx * sl2;
          const bool need = off && ms > -INFINITY;
          // with nothing summed yet the reference may move anywhere; else it
          // drops by at most 2^126 (the earlier keys, p >= 2^-126 against the
          // old reference, then dominate), so alpha stays finite
          const float m_new = !need ? m_ref : (l > 0.f ? fmaxf(ms, m_ref - 126.f) : ms);
          const float alpha = (need && l > 0.f) ? lf_ex2(m_ref - m_new) : 1.f;
          l *= alpha;
          if (t >= 1 && __any_sync(0xffffffffu, need)) {
            gate.pass();  // O holds P.V of the item's earlier tiles, all done
#pragma unroll
            for (int half = 0; half < 2; half++) {
              float ov[32];
              lf_tmem_ld32(tO + 32 * half, ov);
#pragma unroll
              for (int kk = 0; kk < 32; kk++) ov[kk] *= alpha;
              lf_tmem_st32(tO + 32 * half, ov);
            }
          }
          m_ref = m_new;
          lf_tile_pass<kF16>(tS, tP, w, sl2, m_ref, lt, mx, false, gate);
        }
        l += lt;
        gate.pass();  // (no-op unless every chunk of the tile was skipped)
        lf_tmem_wait_st();
        lf_tc_fence_before();
        __syncwarp();
        if (lane == 0) lf_mbar_arrive(p_full);
      }
      if (!alive) break;
      Ctx nxt;
      const int nst = setup(k + 1, nxt);
      if (nst < 0) {
        alive = false;
        break;
      }
      // ---- item epilogue: O / l and the log-normaliser
      if (!lf_wait_warp(o_full, k & 1, abort_flag, D.status, 9)) {
        alive = false;
        break;
      }
      lf_tc_fence_after();
      uint32_t ra[32], rb[32];
      lf_tmem_ld32_nowait(tO, ra);
      lf_tmem_ld32_nowait(tO + 32, rb);
      lf_tmem_wait_ld_regs(ra);
      lf_tmem_pin_regs(rb);
      // O fully read: the stream's next item may overwrite it
      lf_tc_fence_before();
      __syncwarp();
      if (lane == 0) lf_mbar_arrive(o_free);
      const size_t bh = (size_t)it.b * D.H + it.h;
      const bool store_row = it.gitem ? active : (it.qrow0 + q < it.cnt && code != 2);
      if (store_row) {
        if (it.gitem) {
          const size_t pi = (bh * D.G + (it.qrow0 + q)) * D.nch + (it.kt0 / D.chunk_tiles);
          float4 *dst = reinterpret_cast<float4 *>(P.part_acc + pi * LF_HD);
#pragma unroll
          for (int kk = 0; kk < 8; kk++)
            dst[kk] = make_float4(__uint_as_float(ra[4 * kk]), __uint_as_float(ra[4 * kk + 1]),
                                  __uint_as_float(ra[4 * kk + 2]), __uint_as_float(ra[4 * kk + 3]));
#pragma unroll
          for (int kk = 0; kk < 8; kk++)
            dst[8 + kk] = make_float4(__uint_as_float(rb[4 * kk]), __uint_as_float(rb[4 * kk + 1]),
                                      __uint_as_float(rb[4 * kk + 2]), __uint_as_float(rb[4 * kk + 3]));
          P.part_ml[pi] = make_float2(m_ref, l);
        } else {
          const float inv = (code == 1 && l > 0.f) ? 1.f / l : 0.f;
          const size_t orow = bh * n + pos;
          uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<uint16_t *>(P.o) + orow * LF_HD);
#pragma unroll
          for (int kk = 0; kk < 4; kk++) {
            uint4 u;
            u.x = lf_pack2<kF16>(__uint_as_float(ra[8 * kk + 0]) * inv, __uint_as_float(ra[8 * kk + 1]) * inv);
            u.y = lf_pack2<kF16>(__uint_as_float(ra[8 * kk + 2]) * inv, __uint_as_float(ra[8 * kk + 3]) * inv);
            u.z = lf_pack2<kF16>(__uint_as_float(ra[8 * kk + 4]) * inv, __uint_as_float(ra[8 * kk + 5]) * inv);
            u.w = lf_pack2<kF16>(__uint_as_float(ra[8 * kk + 6]) * inv, __uint_as_float(ra[8 * kk + 7]) * inv);
            dst[kk] = u;
          }
#pragma unroll
          for (int kk = 0; kk < 4; kk++) {
            uint4 u;
            u.x = lf_pack2<kF16>(__uint_as_float(rb[8 * kk + 0]) * inv, __uint_as_float(rb[8 * kk + 1]) * inv);
            u.y = lf_pack2<kF16>(__uint_as_float(rb[8 * kk + 2]) * inv, __uint_as_float(rb[8 * kk + 3]) * inv);
            u.z = lf_pack2<kF16>(__uint_as_float(rb[8 * kk + 4]) * inv, __uint_as_float(rb[8 * kk + 5]) * inv);
            u.w = lf_pack2<kF16>(__uint_as_float(rb[8 * kk + 6]) * inv, __uint_as_float(rb[8 * kk + 7]) * inv);
            dst[4 + kk] = u;
          }
          if (P.lse) P.lse[orow] = code == 1 ? (m_ref + __log2f(l)) * LF_LN2 : -INFINITY;
        }
      }
      k++;
      gt += it.T;
      cur = nxt;
      st = nst;
    }
    lf_tmem_wait_st();  // (an abort may leave P stores in flight)
  }

  // ---------------------------------------------------- teardown
  lf_tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    lf_tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(LF_TM_COLS)
                 : "memory");
  }
}
// ------------------------------------------------------------ gather / combine

// Compact, per (b, h), the Q_g rows (global queries) and the K_s / V_s rows
// (global keys for the band's global columns) of the global tokens; rows
// past the sequence's global count are zero.
template <typename T>
__global__ void __launch_bounds__(256)
    lf_gather_kernel(LfDev D, const T *qg, const T *ks, const T *vs, T *qg_c, T *ks_c, T *vs_c,
                     int Ga, int Gka) {
  const int lane = threadIdx.x & 31;
  const long long w = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const long long total = (long long)D.B * D.H * Gka;
  if (w >= total) return;
  const int e = (int)(w % Gka);
  const long long bh = w / Gka;
  const int b = (int)(bh / D.H);
  const int ng = D.binfo[(size_t)b * LF_BI_WORDS + LF_BI_NG];
  uint32_t q = 0, k = 0, v = 0;
  if (e < ng) {
    const int g = D.gidx[(size_t)b * D.G + e];
    const size_t src = ((size_t)bh * D.n + g) * LF_HD + 2 * lane;
    q = *reinterpret_cast<const uint32_t *>(qg + src);
    k = *reinterpret_cast<const uint32_t *>(ks + src);
    v = *reinterpret_cast<const uint32_t *>(vs + src);
  }
  if (e < Ga) *reinterpret_cast<uint32_t *>(qg_c + ((size_t)bh * Ga + e) * LF_HD + 2 * lane) = q;
  *reinterpret_cast<uint32_t *>(ks_c + ((size_t)bh * Gka + e) * LF_HD + 2 * lane) = k;
  *reinterpret_cast<uint32_t *>(vs_c + ((size_t)bh * Gka + e) * LF_HD + 2 * lane) = v;
}

// Merge the split-KV partials of every global row: o = sum_c acc_c 2^(m_c-m)
// / sum_c l_c 2^(m_c-m), lse = (m + log2 sum) ln 2.
template <typename T>
__global__ void __launch_bounds__(256)
    lf_combine_kernel(LfDev D, const float *part_acc, const float2 *part_ml, T *o, float *lse) {
  asm volatile("griddepcontrol.wait;" ::: "memory");  // the partials of the forward kernel
  const int lane = threadIdx.x & 31;
  const long long w = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (w >= (long long)D.B * D.H * D.G) return;
  const int e = (int)(w % D.G);
  const long long bh = w / D.G;
  const int b = (int)(bh / D.H);
  const int ng = D.binfo[(size_t)b * LF_BI_WORDS + LF_BI_NG];
  if (e >= ng) return;
  const size_t base = ((size_t)bh * D.G + e) * D.nch;
  // the output row: the global token's position, or (cross-attention) the query row
  const size_t orow = D.cross ? (size_t)bh * D.G + e : (size_t)bh * D.n + D.gidx[(size_t)b * D.G + e];
  float m = -INFINITY;
  for (int c = 0; c < D.nch; c++) m = fmaxf(m, part_ml[base + c].x);
  float L = 0.f, a0 = 0.f, a1 = 0.f;
  for (int c = 0; c < D.nch; c++) {
    const float2 ml = part_ml[base + c];
    if (ml.y == 0.f) continue;
    const float f = exp2f(ml.x - m);
    L += ml.y * f;
    const float2 acc = *reinterpret_cast<const float2 *>(part_acc + (base + c) * LF_HD + 2 * lane);
    a0 += acc.x * f;
    a1 += acc.y * f;
  }
  // a row with no valid key (cross-attention with every key masked): 0, -inf
  const float inv = L > 0.f ? 1.f / L : 0.f;
  LfIo<T>::st2(o + orow * LF_HD + 2 * lane, a0 * inv, a1 * inv);
  if (lse && lane == 0) lse[orow] = L > 0.f ? (m + log2f(L)) * LF_LN2 : -INFINITY;
}

// ------------------------------------------------------------ host side

static PFN_cuTensorMapEncodeTiled lf_encode_fn() {
  static PFN_cuTensorMapEncodeTiled fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (PFN_cuTensorMapEncodeTiled)p;
  }
  return fn;
}

// 4-D tiled map over rows of 64 elements: dims {64, rows, H, B}; strides in
// bytes {row_stride, head_stride, batch_stride}; box {64, box_rows, 1, 1}.
bool lf_make_map(CUtensorMap *m, int f16, const void *base, uint64_t rows, uint64_t H,
                        uint64_t B, uint64_t row_stride, uint64_t head_stride,
                        uint64_t batch_stride, uint32_t box_rows) {
  PFN_cuTensorMapEncodeTiled enc = lf_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[4] = {64, rows, H, B};
  cuuint64_t strides[3] = {row_stride, head_stride, batch_stride};
  cuuint32_t box[4] = {64, box_rows, 1, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  CUresult r = enc(m, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
                   const_cast<void *>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

cudaError_t lf_launch_gather(const LfLaunch &L, const void *qg, const void *ks, const void *vs,
                             void *qg_c, void *ks_c, void *vs_c, int Ga, int Gka) {
  const LfDev &D = L.dev;
  const long long rows = (long long)D.B * D.H * Gka;
  const unsigned grid = (unsigned)((rows + 7) / 8);
  if (L.dtype == LF_F16)
    lf_gather_kernel<__half><<<grid, 256, 0, L.stream>>>(D, (const __half *)qg, (const __half *)ks,
                                                         (const __half *)vs, (__half *)qg_c,
                                                         (__half *)ks_c, (__half *)vs_c, Ga, Gka);
  else
    lf_gather_kernel<__nv_bfloat16><<<grid, 256, 0, L.stream>>>(
        D, (const __nv_bfloat16 *)qg, (const __nv_bfloat16 *)ks, (const __nv_bfloat16 *)vs,
        (__nv_bfloat16 *)qg_c, (__nv_bfloat16 *)ks_c, (__nv_bfloat16 *)vs_c, Ga, Gka);
  lf_launches_add(1);
  return cudaGetLastError();
}

// Launch with programmatic stream serialization: the kernel may start while
// the previous kernel on the stream finishes, and waits for it (griddepcontrol)
// before reading its results.
static cudaError_t lf_launch_pdl_args(const void *fn, unsigned grid, unsigned block, size_t smem,
                                      cudaStream_t stream, void **args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelExC(&cfg, fn, args);
}
static cudaError_t lf_launch_pdl(const void *fn, unsigned grid, unsigned block, size_t smem,
                                 cudaStream_t stream, LfTcParams *P) {
  void *args[] = {(void *)P};
  return lf_launch_pdl_args(fn, grid, block, smem, stream, args);
}

int lf_tc_fwd(const LfLaunch &L, const LfTcArgs &a, char *err, size_t errlen) {
  const LfDev &D = L.dev;
  const int f16 = L.dtype == LF_F16 ? 1 : 0;
  LfTcParams P;  // host staging; the launch copies the parameter block
  memset(&P, 0, sizeof(P));
  P.dev = D;
  P.f16 = f16;
  const uint64_t n = D.n, H = D.H, B = D.B, rowb = 128;
  int nmaps = 0;
  // segments: runs of heads with equal dilation x residues
  std::map<std::pair<int, int>, int> rmap;
  int nseg = 0, start = 0;
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
        if (nmaps + 3 > LF_TC_MAX_MAPS - 5) goto too_big;
        const char *srcs[3] = {(const char *)a.qs, (const char *)a.ks, (const char *)a.vs};
        for (int k = 0; k < 3; k++)
          if (!lf_make_map(&P.maps[nmaps + k], f16, srcs[k] + rho * rowb, cnt, H, B, d * rowb,
                           n * rowb, H * n * rowb, LF_BQ)) {
            snprintf(err, errlen, "tensor map encode failed (d=%d, rho=%d)", d, rho);
            return LF_ERR_CUDA;
          }
        rmap[key] = nmaps;
        nmaps += 3;
      }
      if (nseg >= LF_TC_MAX_SEG) goto too_big;
      P.seg[nseg] = LfTcSeg{h0, h1, d, rho, cnt, nqb, start, rmap[key]};
      start += (h1 - h0) * nqb;
      nseg++;
    }
    h0 = h1;
  }
  P.nseg = nseg;
  P.per_batch = start;
  {
    // global-row (split-KV) maps and the compacted global-token rows
    const int G = D.G;
    const size_t eb = 2;
    const int Ga = L.ws.G, Gka = L.ws.Gk;
    char *qg_c = L.ws_base + L.ws.qg_c, *ks_c = L.ws_base + L.ws.ks_c, *vs_c = L.ws_base + L.ws.vs_c;
    P.map_kg = nmaps;
    P.map_vg = nmaps + 1;
    P.map_qgc = nmaps + 2;
    P.map_ksc = nmaps + 3;
    P.map_vsc = nmaps + 4;
    P.gbox = std::min(Gka, LF_BK);
    bool ok = lf_make_map(&P.maps[nmaps], f16, a.kg, n, H, B, rowb, n * rowb, H * n * rowb, LF_BK) &&
              lf_make_map(&P.maps[nmaps + 1], f16, a.vg, n, H, B, rowb, n * rowb, H * n * rowb, LF_BK) &&
              lf_make_map(&P.maps[nmaps + 2], f16, qg_c, Ga, H, B, rowb, Ga * rowb, H * Ga * rowb, LF_BQ) &&
              lf_make_map(&P.maps[nmaps + 3], f16, ks_c, Gka, H, B, rowb, Gka * rowb, H * Gka * rowb, P.gbox) &&
              lf_make_map(&P.maps[nmaps + 4], f16, vs_c, Gka, H, B, rowb, Gka * rowb, H * Gka * rowb, P.gbox);
    if (!ok) {
      snprintf(err, errlen, "tensor map encode failed (global maps)");
      return LF_ERR_CUDA;
    }
    nmaps += 5;
    P.ngq = (G + LF_BQ - 1) / LF_BQ;
    P.n_gitems = G > 0 ? D.B * D.H * P.ngq * D.nch : 0;
    P.o = a.o;
    P.lse = a.lse;
    P.part_acc = (float *)(L.ws_base + L.ws.part_acc);
    P.part_ml = (float2 *)(L.ws_base + L.ws.part_ml);
    (void)eb;
    // the mask pass (global list, rank array, sequence info, input checks),
    // fused with the compaction of the global tokens' rows when the list
    // fits in shared memory
    cudaError_t e;
    if (G > 0 && G <= 8192) {  // list in shared memory: 32 KB at most
      e = lf_launch_mask_gather(L, a.qg, a.ks, a.vs, qg_c, ks_c, vs_c, Ga, Gka);
    } else {
      e = lf_launch_mask_pass(L);
      if (e == cudaSuccess && G > 0) e = lf_launch_gather(L, a.qg, a.ks, a.vs, qg_c, ks_c, vs_c, Ga, Gka);
    }
    if (e != cudaSuccess) {
      snprintf(err, errlen, "mask pass / gather launch: %s", cudaGetErrorString(e));
      return LF_ERR_CUDA;
    }
  }
  {
    void (*kern)(const LfTcParams) = f16 ? lf_tc_fwd_kernel<1> : lf_tc_fwd_kernel<0>;
    {
      cudaError_t e = lf_kernel_smem((const void *)kern, LF_SMEM_BYTES);  // per device
      if (e != cudaSuccess) {
        snprintf(err, errlen, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
        return LF_ERR_CUDA;
      }
    }
    const long long items = (long long)P.n_gitems + (long long)D.B * P.per_batch;
    // persistent: one CTA per SM
    const unsigned grid = (unsigned)std::max<long long>(1, std::min<long long>(items, lf_sm_count()));
    P.sched_cta = items <= 4LL * grid ? 1 : 0;
    if (a.ev_start && a.ev_stop) cudaEventRecord(a.ev_start, L.stream);
    cudaError_t le = lf_launch_pdl((const void *)kern, grid, LF_TC_THREADS, LF_SMEM_BYTES, L.stream, &P);
    lf_launches_add(1);
    if (a.ev_start && a.ev_stop) cudaEventRecord(a.ev_stop, L.stream);
    cudaError_t e = le != cudaSuccess ? le : cudaGetLastError();
    if (e != cudaSuccess) {
      snprintf(err, errlen, "tensor-core forward launch: %s", cudaGetErrorString(e));
      return LF_ERR_CUDA;
    }
  }
  if (D.G > 0) {
    const long long rows = (long long)D.B * D.H * D.G;
    const unsigned grid = (unsigned)((rows + 7) / 8);
    const float *pacc = (const float *)P.part_acc;
    const float2 *pml = (const float2 *)P.part_ml;
    cudaError_t le;
    if (f16) {
      __half *o = (__half *)a.o;
      void *args[] = {(void *)&D, (void *)&pacc, (void *)&pml, (void *)&o, (void *)&a.lse};
      le = lf_launch_pdl_args((const void *)lf_combine_kernel<__half>, grid, 256, 0, L.stream, args);
    } else {
      __nv_bfloat16 *o = (__nv_bfloat16 *)a.o;
      void *args[] = {(void *)&D, (void *)&pacc, (void *)&pml, (void *)&o, (void *)&a.lse};
      le = lf_launch_pdl_args((const void *)lf_combine_kernel<__nv_bfloat16>, grid, 256, 0, L.stream, args);
    }
    lf_launches_add(1);
    cudaError_t e = le != cudaSuccess ? le : cudaGetLastError();
    if (e != cudaSuccess) {
      snprintf(err, errlen, "combine launch: %s", cudaGetErrorString(e));
      return LF_ERR_CUDA;
    }
  }
  return LF_OK;

too_big:
  // more (dilation, residue) views than one parameter block holds
  snprintf(err, errlen, "tensor-core path: too many distinct dilation residues (sum of distinct "
                        "dilations must stay <= %d)", (LF_TC_MAX_MAPS - 5) / 3);
  return LF_ERR_UNSUPPORTED;
}

// ------------------------------------------------------------ cross-attention

// One block per sequence b: the sequence info the global-row work items read
// (number of query rows, valid keys = key_mask != 0, or all when no mask).
__global__ void __launch_bounds__(256) lf_cross_setup_kernel(LfDev D) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int b = blockIdx.x;
  if (b == 0 && threadIdx.x == 0) D.status[LF_ST_SCHED] = 0;  // the forward's work-item counter
  int c = 0;
  if (D.mask) {
    const int32_t *m = D.mask + (size_t)b * D.n;
    for (int j = threadIdx.x; j < D.n; j += blockDim.x) c += m[j] != 0;
  } else if (threadIdx.x == 0) {
    c = D.n;
  }
  __shared__ int s_c;
  if (threadIdx.x == 0) s_c = 0;
  __syncthreads();
  atomicAdd(&s_c, c);
  __syncthreads();
  if (threadIdx.x == 0) {
    int32_t *bi = D.binfo + (size_t)b * LF_BI_WORDS;
    bi[LF_BI_NG] = D.G;
    bi[LF_BI_NVALID] = s_c;
    bi[LF_BI_GMIN] = 0;
    bi[LF_BI_GMAX] = D.G - 1;
  }
}

cudaError_t lf_launch_cross_setup(const LfLaunch &L) {
  lf_cross_setup_kernel<<<L.dev.B, 256, 0, L.stream>>>(L.dev);
  lf_launches_add(1);
  return cudaGetLastError();
}

int lf_tc_cross_fwd(const LfLaunch &L, const void *q, const void *k, const void *v, void *o,
                    float *lse, cudaEvent_t ev_start, cudaEvent_t ev_stop, char *err, size_t errlen) {
  const LfDev &D = L.dev;
  const int f16 = L.dtype == LF_F16 ? 1 : 0;
  LfTcParams P;
  memset(&P, 0, sizeof(P));
  P.dev = D;
  P.f16 = f16;
  const uint64_t H = D.H, B = D.B, rowb = 128;
  // every work item is a global-row item: 128 query rows x one key chunk
  P.nseg = 0;
  P.per_batch = 0;
  P.map_kg = 0;
  P.map_vg = 1;
  P.map_qgc = 2;
  P.map_ksc = 0;  // (global-column tiles do not occur)
  P.map_vsc = 1;
  P.gbox = LF_BK;
  const uint64_t Lk = D.n, Lq = D.G;
  if (!lf_make_map(&P.maps[0], f16, k, Lk, H, B, rowb, Lk * rowb, H * Lk * rowb, LF_BK) ||
      !lf_make_map(&P.maps[1], f16, v, Lk, H, B, rowb, Lk * rowb, H * Lk * rowb, LF_BK) ||
      !lf_make_map(&P.maps[2], f16, q, Lq, H, B, rowb, Lq * rowb, H * Lq * rowb, LF_BQ)) {
    snprintf(err, errlen, "cross-attention: tensor map encode failed");
    return LF_ERR_CUDA;
  }
  P.ngq = (D.G + LF_BQ - 1) / LF_BQ;
  P.n_gitems = D.B * D.H * P.ngq * D.nch;
  P.o = o;
  P.lse = lse;
  P.part_acc = (float *)(L.ws_base + L.ws.part_acc);
  P.part_ml = (float2 *)(L.ws_base + L.ws.part_ml);
  cudaError_t e = lf_launch_cross_setup(L);
  if (e != cudaSuccess) {
    snprintf(err, errlen, "cross setup launch: %s", cudaGetErrorString(e));
    return LF_ERR_CUDA;
  }
  void (*kern)(const LfTcParams) = f16 ? lf_tc_fwd_kernel<1> : lf_tc_fwd_kernel<0>;
  if ((e = lf_kernel_smem((const void *)kern, LF_SMEM_BYTES)) != cudaSuccess) {
    snprintf(err, errlen, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    return LF_ERR_CUDA;
  }
  const long long items = P.n_gitems;
  const unsigned grid = (unsigned)std::max<long long>(1, std::min<long long>(items, lf_sm_count()));
  P.sched_cta = items <= 4LL * grid ? 1 : 0;
  if (ev_start && ev_stop) cudaEventRecord(ev_start, L.stream);
  cudaError_t le = lf_launch_pdl((const void *)kern, grid, LF_TC_THREADS, LF_SMEM_BYTES, L.stream, &P);
  lf_launches_add(1);
  if (ev_start && ev_stop) cudaEventRecord(ev_stop, L.stream);
  e = le != cudaSuccess ? le : cudaGetLastError();
  if (e != cudaSuccess) {
    snprintf(err, errlen, "cross-attention launch: %s", cudaGetErrorString(e));
    return LF_ERR_CUDA;
  }
  const long long rows = (long long)D.B * D.H * D.G;
  const unsigned cgrid = (unsigned)((rows + 7) / 8);
  const float *pacc = (const float *)P.part_acc;
  const float2 *pml = (const float2 *)P.part_ml;
  if (f16) {
    __half *oo = (__half *)o;
    void *args[] = {(void *)&D, (void *)&pacc, (void *)&pml, (void *)&oo, (void *)&lse};
    le = lf_launch_pdl_args((const void *)lf_combine_kernel<__half>, cgrid, 256, 0, L.stream, args);
  } else {
    __nv_bfloat16 *oo = (__nv_bfloat16 *)o;
    void *args[] = {(void *)&D, (void *)&pacc, (void *)&pml, (void *)&oo, (void *)&lse};
    le = lf_launch_pdl_args((const void *)lf_combine_kernel<__nv_bfloat16>, cgrid, 256, 0, L.stream, args);
  }
  lf_launches_add(1);
  e = le != cudaSuccess ? le : cudaGetLastError();
  if (e != cudaSuccess) {
    snprintf(err, errlen, "combine launch: %s", cudaGetErrorString(e));
    return LF_ERR_CUDA;
  }
  return LF_OK;
}


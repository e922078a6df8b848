// lf_tc.cu -- tensor-core (tcgen05 / TMEM / TMA) forward of Longformer
// attention for sm_100a, bf16 or f16 inputs, fp32 accumulation.
//
// One persistent kernel (one CTA per SM) runs two kinds of work items:
//
//  * BAND items: 128 query rows t0..t0+127 of one (b, h, residue rho).  A
//    head with dilation d is split into its d residue sub-sequences
//    rho, rho+d, ... ("gaps of size d": segmentfault page, section
//    扩张滑动窗口); in sub-sequence coordinates the window is a plain band of
//    radius r (causal: [t-r, t]), so the item walks only the 128-key tiles
//    that meet the band and the sequence (page section 实现: only a fixed
//    number of diagonals of QK^T are computed).  The residue view is a TMA
//    tensor map whose row stride is d rows, so dilated heads need no gather.
//    After the band tiles come the global-column tiles: the K_s / V_s rows
//    of the sequence's global tokens, fetched with TMA row gathers, minus the
//    keys already inside the row's window (the union of the glossary
//    example), merged into the same online softmax.  Global query rows are
//    skipped (their output comes from the global items); mask-0 rows get
//    o = 0, lse = -inf.
//  * GLOBAL items: up to 128 global query rows (Q_g rows gathered by TMA)
//    against a chunk of LF_TC_CHUNK_TILES key tiles of K_g / V_g (every valid
//    key: global attention sees the whole sequence, segmentfault page
//    section 全局注意力).  Each writes an unnormalised partial (acc, max,
//    sum); the CTA that writes the last partial of a row group merges them
//    (split-KV, no separate launch).
//
// Roles of the 512 threads:
//   warps 0-3, 4-7   softmax groups 0 and 1.  The key tiles of an item
//                    alternate between the groups (tile j of the CTA's tile
//                    stream goes to group j & 1), so the two groups work on
//                    the same 128 rows; each has its own S, P and O in TMEM
//                    and its own running reference and sum.  One TMEM lane =
//                    one query row per thread.
//   warps 8-11       epilogue: merges the two groups' (O, reference, sum) of
//                    an item, writes O / lse (band) or the split partial and,
//                    for the last partial of a row group, the merged global
//                    rows.
//   warp 12          producer: takes work items from a grid-wide counter
//                    (largest first), issues the TMA loads (Q, K/V ring).
//   warps 13, 14     MMA issuers, one per softmax group: S(j + 2) as soon
//                    as group w = j & 1 has turned S(j) into P(j), then
//                    O_w += P(j) V_j.
//   warp 15          context: per item, the rows' mask codes and window
//                    ranks and the validity bits of the walked keys, in
//                    shared memory, one item ahead of the softmax groups.
// Per tile j (group w = j & 1):
//   softmax  attend mask of the row for the tile (from the item context)
//   MMA      S_w = Q K_j^T                                 -> s_full[w]
//   softmax  P_w = exp2(S*scale*log2e - m) against the row's running
//            reference m (the tile is redone with its own max, O_w rescaled,
//            when the row sum leaves the P format's safe range), row sum
//                                                          -> p_full[w]
//   MMA      S_w = Q K_{j+2}^T; O_w (+)= P_w V_j           -> pv_done[w]
// The n x w score band never leaves the SM.
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

#define LF_F_THREADS 512
#define LF_FK 64           // keys per tile
#define LF_F_NS 10         // K/V ring stages (one 64-key tile of K and V each)
#define LF_F_SLOTS 4       // work-item ring slots
#define LF_F_MAX_MAPS 192  // tensor maps in the parameter block
#define LF_F_MAX_SEG 96
#define LF_F_CTX_WORDS 256  // validity / residue bit words of one item context

// TMEM columns: group w has two S buffers (64 columns each; P is written
// over the first 32 columns of the S it came from, bf16/f16 pairs, the A
// operand of P.V) and two O accumulators (item parity)
#define LF_TM_S(w, b) ((w)*128 + (b)*64)
#define LF_TM_O(w, p) (256 + (w)*128 + (p)*64)
#define LF_TM_COLS 512

// Context of one work item (shared memory; built by the context warp).
struct LfCtx {
  int idx;  // work item, -1: no more items
  int gitem, b, h, d, rho, cnt, qrow0, T, nbw, u_lo, nglob, ng, ngk, kt0, tk0;
  int direct;  // 1: the bits did not fit vw; the softmax reads mask / list itself
  int rw0;     // first residue word in vw
  int pad[14];
  int code[128];  // row's mask value; -1: no row (past the sub-sequence / the global list)
  int pos[128];   // row's sequence position
  int elo[128], ehi[128];  // global keys inside the row's window: list range [elo, ehi)
  uint32_t vw[LF_F_CTX_WORDS];  // validity bits of the walked keys, then residue bits
};
static_assert(sizeof(LfCtx) % 16 == 0, "context size");

// shared memory map (bytes from the 1024-aligned base)
#define LF_SM_Q(p) ((p)*16384)
#define LF_SM_K(s) (32768 + (s)*16384)
#define LF_SM_V(s) (32768 + (s)*16384 + 8192)
#define LF_SM_CTX (32768 + LF_F_NS * 16384)
#define LF_SM_ML (LF_SM_CTX + 2 * (int)sizeof(LfCtx))
#define LF_SM_BAR (LF_SM_ML + 2 * 2 * 128 * 8)
#define LF_NBAR 64
#define LF_SM_MISC (LF_SM_BAR + LF_NBAR * 8)
#define LF_SMEM_BYTES (LF_SM_MISC + 256)
static_assert(LF_SMEM_BYTES <= 232448, "shared memory per CTA");

// barrier indices
#define LB_IT_FULL(i) (i)
#define LB_IT_EMPTY(i) (4 + (i))
#define LB_CTX_FULL(p) (8 + (p))
#define LB_CTX_EMPTY(p) (10 + (p))
#define LB_Q_FULL(p) (12 + (p))
#define LB_Q_EMPTY(p) (14 + (p))
#define LB_S_FULL(w, b) (16 + 2 * (w) + (b))
#define LB_P_FULL(w, b) (20 + 2 * (w) + (b))
#define LB_PV_DONE(w) (24 + (w))
#define LB_ML_FULL(p) (26 + (p))
#define LB_ML_EMPTY(p) (28 + (p))
#define LB_O_FULL(p) (30 + (p))
#define LB_O_FREE(p) (32 + (p))
#define LB_EPI 34
#define LB_END(w) (35 + (w))
#define LB_STAGGER 37
#define LB_KV_FULL(s) (40 + (s))
#define LB_KV_EMPTY(s) (50 + (s))
static_assert(LF_F_NS <= 10, "kv barriers");

// One run of heads with equal dilation x one residue sub-sequence.  Its
// 128-row blocks are split into interior blocks (the full band inside the
// sub-sequence) and edge blocks (nl at the start, nr at the end), which are
// cheaper and scheduled last.
struct LfFSeg {
  int h0, h1, d, rho, cnt, nqb, nl, nr, start1, start2, map;
};

struct LfFwdParams {
  CUtensorMap maps[LF_F_MAX_MAPS];
  LfDev dev;
  LfFSeg seg[LF_F_MAX_SEG];
  int nseg, per1, per2, n_gitems, ngq;
  int map_kg, map_vg, map_qg2, map_ks2, map_vs2;
  void *o;
  float *lse;
  float *part_acc;
  float2 *part_ml;
  int *gcount;
};

// max of three floats (sm_100 three-input max)
__device__ __forceinline__ float lf_max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Masks one 32-column chunk of raw scores in place (columns whose bit in
// wc is clear become -inf) and returns its max.
__device__ __forceinline__ float lf_mask_max(uint32_t (&x)[32], uint32_t wc) {
  if (!__all_sync(0xffffffffu, wc == 0xffffffffu)) {
#pragma unroll
    for (int k = 0; k < 32; k++) x[k] = ((wc >> k) & 1u) ? x[k] : 0xff800000u;  // -inf
  }
  float m0 = __uint_as_float(x[0]), m1 = __uint_as_float(x[1]);
#pragma unroll
  for (int k = 2; k < 30; k += 4) {
    m0 = lf_max3(m0, __uint_as_float(x[k]), __uint_as_float(x[k + 1]));
    m1 = lf_max3(m1, __uint_as_float(x[k + 2]), __uint_as_float(x[k + 3]));
  }
  return lf_max3(m0, m1, fmaxf(__uint_as_float(x[30]), __uint_as_float(x[31])));
}

// P of one masked 32-column chunk against the reference (mneg = -m):
// p = 2^(s*sl2 - m), written as 16-bit pairs to TMEM at tP (16 columns),
// summed into s0 / s1.  A chunk no lane attends is written as zeros.
template <int kF16>
__device__ __forceinline__ void lf_p_chunk(const uint32_t (&x)[32], bool anyc, float sl2,
                                           float mneg, uint32_t tP, float &s0, float &s1) {
  if (!anyc) {
#pragma unroll
    for (int g = 0; g < 4; g++) lf_tmem_st4(tP + 4 * g, 0u, 0u, 0u, 0u);
    return;
  }
  // four pieces of 8 values (4 packed columns): few registers live at once
#pragma unroll
  for (int g = 0; g < 4; g++) {
    uint32_t pw[4];
#pragma unroll
    for (int k = 0; k < 8; k += 2) {
      const float p0 = lf_ex2(fmaf(__uint_as_float(x[8 * g + k]), sl2, mneg));
      const float p1 = lf_ex2(fmaf(__uint_as_float(x[8 * g + k + 1]), sl2, mneg));
      s0 += p0;
      s1 += p1;
      pw[k / 2] = lf_pack2<kF16>(p0, p1);
    }
    lf_tmem_st4(tP + 4 * g, pw[0], pw[1], pw[2], pw[3]);
  }
}

// O *= alpha for this thread's TMEM lane (64 columns), 8 columns at a time;
// out of line: it runs only when a row's max grew by more than 2^8.
static __device__ __noinline__ void lf_rescale_o(uint32_t tO, float alpha) {
#pragma unroll 1
  for (int part = 0; part < 8; part++) {
    float ov[8];
    lf_tmem_ld8(tO + 8 * part, ov);
#pragma unroll
    for (int kk = 0; kk < 8; kk++) ov[kk] *= alpha;
    lf_tmem_st8(tO + 8 * part, ov);
  }
}

// A decoded work item (producer, MMA and context warps decode the same way).
struct LfFItem {
  int gitem, b, h, d, rho, cnt, qrow0, T, nbw, u_lo, nglob, ng, ngk, kt0, tk0, map;
};

// Band tiles of 64 keys: tile u of a 128-row block starting at t0 covers
// keys t0 - r + 64u .. +63 (sub-sequence coordinates); the band of row q
// (0..127) is [q, q + span] relative to t0 - r, span = r (causal) or 2r.
__device__ __forceinline__ int lf_f_band_tiles(int r, int causal) {
  return (LF_BQ + (causal ? r : 2 * r) + LF_FK - 1) / LF_FK;
}
__device__ __forceinline__ void lf_f_band_cols(int q, int u, int r, int causal, int &lo, int &hi) {
  const int base = LF_FK * u;
  lo = max(q - base, 0);
  hi = min(q + (causal ? r : 2 * r) - base, LF_FK - 1);
}

__device__ __forceinline__ bool lf_fdecode(const LfFwdParams &P, int idx, LfFItem &it) {
  const LfDev &D = P.dev;
  const int n = D.n;
  it.d = 1;
  it.rho = 0;
  it.cnt = n;
  it.kt0 = 0;
  it.nglob = 0;
  it.u_lo = 0;
  it.map = 0;
  it.ngk = 0;
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
    const int ct = D.chunk_tiles * (LF_BK / LF_FK);  // 64-key tiles per split
    it.kt0 = c * ct;
    const int ktiles = (n + LF_FK - 1) / LF_FK;
    it.nbw = min(ct, ktiles - it.kt0);
    it.T = it.nbw;
    it.tk0 = it.kt0 * LF_FK;
    return it.qrow0 < it.ng && it.nbw > 0;  // false: nothing to do
  }
  it.gitem = 0;
  idx -= P.n_gitems;
  int cls2 = 0, per = P.per1;
  if (idx >= D.B * P.per1) {
    idx -= D.B * P.per1;
    cls2 = 1;
    per = P.per2;
  }
  it.b = idx / per;
  int rem = idx - it.b * per;
  int s = 0;
  if (!cls2) {
    while (s + 1 < P.nseg && rem >= P.seg[s + 1].start1) s++;
    rem -= P.seg[s].start1;
  } else {
    while (s + 1 < P.nseg && rem >= P.seg[s + 1].start2) s++;
    rem -= P.seg[s].start2;
  }
  const LfFSeg &sg = P.seg[s];
  const int nedge = sg.nl + sg.nr, nint = sg.nqb - nedge;
  int qb;
  if (!cls2) {
    it.h = sg.h0 + rem / nint;
    qb = sg.nl + rem % nint;
  } else {
    it.h = sg.h0 + rem / nedge;
    const int e = rem % nedge;
    qb = e < sg.nl ? e : sg.nqb - sg.nr + (e - sg.nl);
  }
  it.qrow0 = qb * LF_BQ;
  it.d = sg.d;
  it.rho = sg.rho;
  it.cnt = sg.cnt;
  it.map = sg.map;
  // band tiles u = 0 .. nband-1; walk those that meet [0, cnt)
  const int nband = lf_f_band_tiles(D.r, D.causal);
  const int base = it.qrow0 - D.r;
  const int x = -base - (LF_FK - 1);
  it.u_lo = x > 0 ? (x + LF_FK - 1) / LF_FK : 0;
  const int u_hi = min(nband, (it.cnt - base + LF_FK - 1) / LF_FK);
  it.nbw = u_hi - it.u_lo;
  it.tk0 = base + LF_FK * it.u_lo;
  const int32_t *bi = D.binfo + (size_t)it.b * LF_BI_WORDS;
  it.ng = bi[LF_BI_NG];
  bool need = it.ng > 0;
  if (need && it.d == 1 && !D.causal) {
    // every global key inside every row's window: the band covers them
    const int tlast = min(it.qrow0 + LF_BQ - 1, it.cnt - 1);
    if (bi[LF_BI_GMIN] >= tlast - D.r && bi[LF_BI_GMAX] <= it.qrow0 + D.r) need = false;
  }
  it.nglob = need ? (it.ng + LF_FK - 1) / LF_FK : 0;
  it.ngk = (it.ng + 15) / 16 * 16;
  it.T = it.nbw + it.nglob;
  return true;
}

// TMA gather of four rows of 64 elements (a 2-D map over [B*H*n, 64] with a
// one-row box) into 512 consecutive bytes of shared memory.
__device__ __forceinline__ void lf_tma_gather4(uint32_t dst, const CUtensorMap *map, uint32_t bar,
                                               int r0, int r1, int r2, int r3) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(0), "r"(r0), "r"(r1), "r"(r2), "r"(r3), "r"(bar)
      : "memory");
}

// ------------------------------------------------------------ the kernel

template <int kF16>
__global__ void __launch_bounds__(LF_F_THREADS, 1)
    lf_tc_fwd_kernel(const __grid_constant__ LfFwdParams P) {
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
  const int nitems = P.n_gitems + D.B * (P.per1 + P.per2);

  auto BAR = [&](int i) -> uint32_t { return sbase + LF_SM_BAR + 8 * i; };
  LfCtx *ctxs = reinterpret_cast<LfCtx *>(gbase + LF_SM_CTX);
  float2 *mls = reinterpret_cast<float2 *>(gbase + LF_SM_ML);  // [parity][group][row]
  uint32_t *tmem_slot = (uint32_t *)(gbase + LF_SM_MISC);
  volatile int *abort_flag = (volatile int *)(gbase + LF_SM_MISC + 4);  // [2]: flag, wait limit
  volatile int *item_slot = (volatile int *)(gbase + LF_SM_MISC + 12);  // [LF_F_SLOTS]
  volatile int *epi_flag = (volatile int *)(gbase + LF_SM_MISC + 28);

  if (threadIdx.x == 0) {
    for (int i = 0; i < LF_F_SLOTS; i++) {
      lf_mbar_init(BAR(LB_IT_FULL(i)), 1);
      lf_mbar_init(BAR(LB_IT_EMPTY(i)), 3);  // two MMA warps + the context warp
    }
    for (int p = 0; p < 2; p++) {
      lf_mbar_init(BAR(LB_CTX_FULL(p)), 1);    // the context warp
      lf_mbar_init(BAR(LB_CTX_EMPTY(p)), 12);  // eight softmax + four epilogue warps
      lf_mbar_init(BAR(LB_Q_FULL(p)), 1);
      lf_mbar_init(BAR(LB_Q_EMPTY(p)), 2);  // both MMA warps, once per item
      lf_mbar_init(BAR(LB_PV_DONE(p)), 1);
      lf_mbar_init(BAR(LB_ML_FULL(p)), 8);   // both groups
      lf_mbar_init(BAR(LB_ML_EMPTY(p)), 4);  // epilogue warps
      lf_mbar_init(BAR(LB_O_FULL(p)), 2);    // both MMA warps, once per item
      lf_mbar_init(BAR(LB_O_FREE(p)), 4);    // epilogue warps
      lf_mbar_init(BAR(LB_END(p)), 1);
      for (int b = 0; b < 2; b++) {
        lf_mbar_init(BAR(LB_S_FULL(p, b)), 1);
        lf_mbar_init(BAR(LB_P_FULL(p, b)), 4);  // the group's four warps
      }
    }
    lf_mbar_init(BAR(LB_EPI), 4);
    lf_mbar_init(BAR(LB_STAGGER), 4);  // group 0's warps, once
    for (int s = 0; s < LF_F_NS; s++) {
      lf_mbar_init(BAR(LB_KV_FULL(s)), 1);
      lf_mbar_init(BAR(LB_KV_EMPTY(s)), 1);
    }
    abort_flag[0] = 0;
    abort_flag[1] = P.dev.wait_us;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 13) {
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
  int32_t *status = D.status;
  if (warp == 12) {
    // ================================================== TMA producer + scheduler
    // the mask pass (launched just before, this kernel is its programmatic
    // dependent) writes the sequence info and the global list read below
    asm volatile("griddepcontrol.wait;" ::: "memory");
    int k = 0, gt = 0;
    bool ok = true;
    // test hook: CTA 0 leaves one K/V stage unloaded, so its consumer's
    // bounded wait expires (LF_ERR_DEVICE_TIMEOUT) and the CTA aborts
    const int skip = (D.skip_tile > 0 && blockIdx.x == 0) ? D.skip_tile - 1 : -1;
    // next work item (largest first: global rows, interior band blocks,
    // edge band blocks), from one grid-wide counter; empty items skipped.
    // Item kk is published into ring slot kk % LF_F_SLOTS.
    auto publish = [&](int kk) -> int {
      int idx = -1;
      if (lane == 0) {
        LfFItem t_;
        for (;;) {
          idx = atomicAdd(status + LF_ST_SCHED, 1);
          if (idx >= nitems) {
            idx = -1;
            break;
          }
          if (lf_fdecode(P, idx, t_)) break;
        }
      }
      idx = __shfl_sync(0xffffffffu, idx, 0);
      const int slot = kk % LF_F_SLOTS;
      if (kk >= LF_F_SLOTS && !lf_wait_warp(BAR(LB_IT_EMPTY(slot)), ((kk / LF_F_SLOTS) & 1) ^ 1,
                                            abort_flag, status, 16))
        return -2;
      if (lane == 0) {
        item_slot[slot] = idx;
        lf_mbar_arrive(BAR(LB_IT_FULL(slot)));
      }
      return idx;
    };
    // one item is published ahead of the one being loaded, so the context
    // warp prepares it while the current item's loads are still going
    int nxt = publish(0);
    while (ok) {
      const int idx = nxt;
      if (idx < 0) break;
      nxt = publish(k + 1);
      if (nxt == -2) break;
      LfFItem it;
      lf_fdecode(P, idx, it);
      const int qp = k & 1;
      const uint32_t qbar = BAR(LB_Q_FULL(qp));
      // the item two back used this Q buffer: all its S products must be done
      if (k >= 2 && !lf_wait_warp(BAR(LB_Q_EMPTY(qp)), ((k >> 1) & 1) ^ 1, abort_flag, status, 1)) {
        ok = false;
        break;
      }
      const size_t bhn = ((size_t)it.b * D.H + it.h) * n;
      const int32_t *gl = D.gidx + (size_t)it.b * D.G;
      if (!it.gitem) {
        if (lane == 0) {
          lf_mbar_expect_tx(qbar, 16384);
          lf_tma_load4(sbase + LF_SM_Q(qp), &P.maps[it.map], qbar, 0, it.qrow0, it.h, it.b);
        }
      } else {
        // the group's global query rows; rows past the list repeat its first row
        const int rows = min(LF_BQ, it.ng - it.qrow0), r4 = (rows + 3) / 4;
        if (lane == 0) lf_mbar_expect_tx(qbar, r4 * 4 * 128);
        __syncwarp();
        if (lane < r4) {
          int rr[4];
#pragma unroll
          for (int i = 0; i < 4; i++) {
            const int e = it.qrow0 + 4 * lane + i;
            rr[i] = (int)(bhn + gl[e < it.ng ? e : it.qrow0]);
          }
          lf_tma_gather4(sbase + LF_SM_Q(qp) + 512 * lane, &P.maps[P.map_qg2], qbar, rr[0], rr[1],
                         rr[2], rr[3]);
        }
      }
      for (int t = 0; t < it.T; t++, gt++) {
        const int s = gt % LF_F_NS;
        if (gt >= LF_F_NS && !lf_wait_warp(BAR(LB_KV_EMPTY(s)), ((gt / LF_F_NS) & 1) ^ 1,
                                           abort_flag, status, 2)) {
          ok = false;
          break;
        }
        const uint32_t kvb = BAR(LB_KV_FULL(s));
        if (gt == skip) continue;
        if (t < it.nbw) {
          if (lane == 0) {
            const int row = it.tk0 + t * LF_FK;
            const CUtensorMap *km = &P.maps[it.gitem ? P.map_kg : it.map + 1];
            const CUtensorMap *vm = &P.maps[it.gitem ? P.map_vg : it.map + 2];
            lf_mbar_expect_tx(kvb, 2 * 8192);
            lf_tma_load4(sbase + LF_SM_K(s), km, kvb, 0, row, it.h, it.b);
            lf_tma_load4(sbase + LF_SM_V(s), vm, kvb, 0, row, it.h, it.b);
          }
        } else {
          // global keys gbs .. gbs + rows - 1 of the list (rows past the list
          // repeat its first entry: finite values at masked columns)
          const int gbs = (t - it.nbw) * LF_FK;
          const int rows = min(LF_FK, it.ngk - gbs), r4 = rows / 4;
          if (lane == 0) lf_mbar_expect_tx(kvb, 2 * rows * 128);
          __syncwarp();
          if (lane < r4) {
            int rr[4];
#pragma unroll
            for (int i = 0; i < 4; i++) {
              const int e = gbs + 4 * lane + i;
              rr[i] = (int)(bhn + gl[e < it.ng ? e : 0]);
            }
            lf_tma_gather4(sbase + LF_SM_K(s) + 512 * lane, &P.maps[P.map_ks2], kvb, rr[0], rr[1],
                           rr[2], rr[3]);
            lf_tma_gather4(sbase + LF_SM_V(s) + 512 * lane, &P.maps[P.map_vs2], kvb, rr[0], rr[1],
                           rr[2], rr[3]);
          }
        }
      }
      k++;
    }
    if (*abort_flag && lane == 0) {
      // let the copies already issued land before the CTA exits (a stage
      // whose load was issued completes its phase; Q likewise)
      for (int i = max(0, gt - LF_F_NS); i < gt; i++)
        if (i != skip) lf_wait_drain(BAR(LB_KV_FULL(i % LF_F_NS)), (i / LF_F_NS) & 1, status, 11);
      for (int kk = max(0, k - 2); kk < k; kk++)
        lf_wait_drain(BAR(LB_Q_FULL(kk & 1)), (kk >> 1) & 1, status, 12);
    }
  } else if (warp == 13 || warp == 14) {
    // ================================================== MMA issuers
    // Tiles form one stream j = 0, 1, ... over the CTA's items; tile j goes
    // to group w = j & 1 as its c = (j >> 1)-th tile, into S buffer c & 1.
    // MMA warp 13 + w issues group w's products only.  S runs two own tiles
    // ahead: once group w has turned S(c) into P(c) (written over S(c)), the
    // warp issues O_w (+)= P(c) V, then S(c + 2) into the same buffer (MMAs
    // of one thread execute in issue order, so P(c) is read first).  Per item both warps
    // commit q_empty (after their last S of it) and o_full (after their last
    // P.V of it), also for items in which they own no tile; a warp enters item
    // k only after Q(k) is loaded (S side) and after the epilogue freed the O
    // buffers of item k - 2 (P.V side), so neither commit can run ahead of the
    // other warp's commit for an earlier item.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int w = warp - 13;
    const uint64_t dq0 = lf_sdesc(sbase + LF_SM_Q(0), 16, 1024);
    const uint64_t dk0 = lf_sdesc(sbase + LF_SM_K(0), 16, 1024);
    const uint64_t dv0 = lf_sdesc(sbase + LF_SM_V(0), 0, 1024);
    const uint32_t id_pv = lf_idesc(kF16, 64, 1);
    // item queue of this warp (shared memory): T, nbw, ngk of item k at [k % 4]
    volatile int *iq = (volatile int *)(gbase + LF_SM_MISC + 64) + 12 * w;
    bool ok = true;
    int nk = 0;  // items taken from the ring
    auto take = [&]() -> bool {
      const int slot = nk % LF_F_SLOTS;
      if (!lf_wait_warp(BAR(LB_IT_FULL(slot)), (nk / LF_F_SLOTS) & 1, abort_flag, status, 15)) {
        ok = false;
        return false;
      }
      const int idx = item_slot[slot];
      __syncwarp();
      if (lane == 0) lf_mbar_arrive(BAR(LB_IT_EMPTY(slot)));
      if (idx < 0) return false;
      LfFItem it;
      lf_fdecode(P, idx, it);
      if (lane == 0) {
        iq[3 * (nk & 3)] = it.T;
        iq[3 * (nk & 3) + 1] = it.nbw;
        iq[3 * (nk & 3) + 2] = it.ngk;
      }
      __syncwarp();
      nk++;
      return true;
    };
    auto qT = [&](int kk) { return iq[3 * (kk & 3)]; };
    auto ncols = [&](int kk, int t) {
      const int nbw = iq[3 * (kk & 3) + 1], ngk = iq[3 * (kk & 3) + 2];
      return t < nbw ? LF_FK : min(LF_FK, ngk - (t - nbw) * LF_FK);
    };
    // S cursor: item sk, tile st of it (stream index sj); ends at s_end
    int sk = 0, st = w, sj = w;
    bool s_end = false;
    // move the S cursor onto an own tile: leave items it has passed
    // (commit q_empty), enter new ones (wait for their Q)
    auto s_settle = [&]() {
      while (!s_end && ok && st >= qT(sk)) {
        st -= qT(sk);
        lf_commit_w(BAR(LB_Q_EMPTY(sk & 1)));  // every S of item sk this warp issues is issued
        sk++;
        if (sk >= nk && !take()) {
          s_end = true;
          break;
        }
        if (!lf_wait_warp(BAR(LB_Q_FULL(sk & 1)), (sk >> 1) & 1, abort_flag, status, 3)) ok = false;
      }
    };
    auto issue_s = [&]() -> bool {
      const int s = sj % LF_F_NS, c = sj >> 1;
      if (!lf_wait_warp(BAR(LB_KV_FULL(s)), (sj / LF_F_NS) & 1, abort_flag, status, 4)) return false;
      lf_tc_fence_after();
      lf_mma_s_phase(tmem + LF_TM_S(w, c & 1), dq0 + (uint64_t)((sk & 1) * (16384 >> 4)),
                     dk0 + (uint64_t)(s * (16384 >> 4)), lf_idesc(kF16, ncols(sk, st), 0),
                     BAR(LB_S_FULL(w, c & 1)));
      st += 2;
      sj += 2;
      s_settle();
      return ok;
    };
    // P.V cursor: leaving an item commits o_full; entering item pk >= 2
    // waits until the epilogue read the O buffers of item pk - 2
    int pk = 0, pt = w, pj = w;
    auto p_settle = [&]() {
      while (ok && pk < nk && pt >= qT(pk)) {
        pt -= qT(pk);
        lf_commit_w(BAR(LB_O_FULL(pk & 1)));  // every P.V of item pk this warp issues is issued
        pk++;
        if (pk < nk && pk >= 2 &&
            !lf_wait_warp(BAR(LB_O_FREE(pk & 1)), ((pk >> 1) & 1) ^ 1, abort_flag, status, 6))
          ok = false;
      }
    };
    if (!take()) {
      s_end = true;
    } else if (lf_wait_warp(BAR(LB_Q_FULL(0)), 0, abort_flag, status, 3)) {
      s_settle();
      for (int i = 0; i < 2 && !s_end && ok; i++) issue_s();
    } else {
      ok = false;
    }
    p_settle();
    while (ok && pk < nk && pj < sj) {
      const int c = pj >> 1, b = c & 1;
      // S(c) consumed and P(c) written over it by group w
      if (!lf_wait_warp(BAR(LB_P_FULL(w, b)), (c >> 1) & 1, abort_flag, status, 5)) {
        ok = false;
        break;
      }
      lf_tc_fence_after();
      const int s = pj % LF_F_NS, nc = ncols(pk, pt);
      lf_mma_ts_phase(tmem + LF_TM_O(w, pk & 1), tmem + LF_TM_S(w, b),
                      dv0 + (uint64_t)(s * (16384 >> 4)), 2048 >> 4, id_pv, (1u << (nc / 16)) - 1u,
                      pt >= 2 ? 1u : 0u, BAR(LB_KV_EMPTY(s)), BAR(LB_PV_DONE(w)), 0u);
      pt += 2;
      pj += 2;
      p_settle();
      if (!s_end && ok) {
        // S(c + 2) goes into buffer b, over P(c): the tensor core executes
        // this thread's MMAs in issue order, so the P.V just issued reads
        // P(c) before this product overwrites it (no wait needed)
        if (!issue_s()) {
          ok = false;
          break;
        }
      }
    }
    // every MMA this warp issued has completed once end_bar flips (waited
    // for also after an abort: TMEM is freed only after that)
    lf_commit_w(BAR(LB_END(w)));
    lf_wait_drain(BAR(LB_END(w)), 0, status, 7);
    __syncwarp();
  } else if (warp == 15) {
    // ================================================== item context
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int tid = lane;
    const int rr = D.r, causal = D.causal;
    for (int k = 0;; k++) {
      const int slot = k % LF_F_SLOTS, par = k & 1;
      if (!lf_wait_warp(BAR(LB_IT_FULL(slot)), (k / LF_F_SLOTS) & 1, abort_flag, status, 17)) break;
      const int idx = item_slot[slot];
      __syncwarp();
      if (lane == 0) lf_mbar_arrive(BAR(LB_IT_EMPTY(slot)));
      if (k >= 2 &&
          !lf_wait_warp(BAR(LB_CTX_EMPTY(par)), ((k >> 1) & 1) ^ 1, abort_flag, status, 18))
        break;
      LfCtx &C = ctxs[par];
      if (idx < 0) {
        if (tid == 0) C.idx = -1;
        __syncwarp();
        if (lane == 0) lf_mbar_arrive(BAR(LB_CTX_FULL(par)));
        break;
      }
      LfFItem it;
      lf_fdecode(P, idx, it);
      const int32_t *mr = D.mask + (size_t)it.b * n;
      const int32_t *gl = D.gidx + (size_t)it.b * D.G;
      const int32_t *gr = D.grank + (size_t)it.b * (n + 1);
      const int nvw = 2 * it.nbw;
      const int nrw = (!it.gitem && it.d > 1 && it.nglob > 0) ? 2 * it.nglob : 0;
      const int direct = nvw + nrw > LF_F_CTX_WORDS ? 1 : 0;
      if (tid == 0) {
        C.idx = idx;
        C.gitem = it.gitem;
        C.b = it.b;
        C.h = it.h;
        C.d = it.d;
        C.rho = it.rho;
        C.cnt = it.cnt;
        C.qrow0 = it.qrow0;
        C.T = it.T;
        C.nbw = it.nbw;
        C.u_lo = it.u_lo;
        C.nglob = it.nglob;
        C.ng = it.ng;
        C.ngk = it.ngk;
        C.kt0 = it.kt0;
        C.tk0 = it.tk0;
        C.direct = direct;
        C.rw0 = nvw;
      }
      // rows tid + 32 i; every load is issued before any result is used
      // (one memory round trip for the codes and the window ranks)
      {
        int code[4], pos[4], elo[4], ehi[4];
#pragma unroll
        for (int i = 0; i < 4; i++) {
          const int q = tid + 32 * i;
          code[i] = -1;
          pos[i] = 0;
          elo[i] = ehi[i] = 0;
          if (it.gitem) {
            const int e = it.qrow0 + q;
            if (e < it.ng) {
              code[i] = 2;
              pos[i] = gl[e];
            }
          } else {
            const int t = it.qrow0 + q;
            if (t < it.cnt) {
              pos[i] = it.rho + t * it.d;
              code[i] = mr[pos[i]];
              if (it.nglob > 0) {  // used by local rows only
                elo[i] = gr[max(pos[i] - rr * it.d, 0)];
                ehi[i] = gr[min((causal ? pos[i] : pos[i] + rr * it.d) + 1, n)];
              }
            }
          }
        }
#pragma unroll
        for (int i = 0; i < 4; i++) {
          const int q = tid + 32 * i;
          C.code[q] = code[i];
          C.pos[q] = pos[i];
          C.elo[q] = elo[i];
          C.ehi[q] = ehi[i];
        }
      }
      if (!direct) {
        // validity of the walked keys (sub-sequence coordinates tk0 + i): one
        // word per thread, its 32 loads issued back to back
        for (int wi = tid; wi < nvw; wi += 32) {
          const int t0 = it.tk0 + 32 * wi;
          uint32_t word = 0;
#pragma unroll
          for (int bit = 0; bit < 32; bit++) {
            const int t = t0 + bit;
            const bool okk = t >= 0 && t < it.cnt && mr[it.rho + t * it.d] != 0;
            word |= (okk ? 1u : 0u) << bit;
          }
          C.vw[wi] = word;
        }
        // global keys of the row's residue (dilated heads)
        for (int wi = tid; wi < nrw; wi += 32) {
          uint32_t word = 0;
#pragma unroll
          for (int bit = 0; bit < 32; bit++) {
            const int e = 32 * wi + bit;
            const bool res = e < it.ng && (gl[e] - it.rho) % it.d == 0;
            word |= (res ? 1u : 0u) << bit;
          }
          C.vw[nvw + wi] = word;
        }
      }
      __syncwarp();
      if (lane == 0) lf_mbar_arrive(BAR(LB_CTX_FULL(par)));
    }
  } else if (warp < 8) {
    // ================================================== softmax groups
    // One flat loop over the group's own tiles of the CTA's tile stream (tile
    // j belongs to group j & 1, its c = (j >> 1)-th, S buffer c & 1), across
    // items.  The TMEM loads of a tile's scores are issued as soon as the
    // previous tile's P is handed over, so their latency overlaps the item
    // bookkeeping and the next tile's attend mask.
    const int grp = warp >> 2, quarter = warp & 3;
    const int q = quarter * 32 + lane;  // query row of the tile == TMEM lane
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const float sl2 = D.scale_log2;
    const int rr = lf_reg(D.r), causal = lf_reg(D.causal);
    // (the direct path below reads the mask pass's global list)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // the current item's fields (registers)
    int k = -1, gt = 0, par = 0, T = 0, gitem = 0, nbw = 0, u_lo = 0, cnt = 0, tk0 = 0, ng = 0,
        dd = 1, direct = 0, e_lo = 0, e_hi = 0;
    bool active = false, has_pv = false, alive = true;
    float m_ref = -INFINITY, l = 0.f;
    uint32_t tO = 0;
    // leave item k: this group's running reference and sum of its rows
    auto leave = [&]() -> bool {
      if (k >= 2 &&
          !lf_wait_warp(BAR(LB_ML_EMPTY(par)), ((k >> 1) & 1) ^ 1, abort_flag, status, 20))
        return false;
      mls[(par * 2 + grp) * 128 + q] = make_float2(m_ref, l);
      __syncwarp();
      if (lane == 0) {
        lf_mbar_arrive(BAR(LB_ML_FULL(par)));
        lf_mbar_arrive(BAR(LB_CTX_EMPTY(par)));
      }
      gt += T;
      return true;
    };
    // enter item k + 1; false when there is none (or the CTA aborted)
    auto enter = [&]() -> bool {
      k++;
      par = k & 1;
      if (!lf_wait_warp(BAR(LB_CTX_FULL(par)), (k >> 1) & 1, abort_flag, status, 19)) {
        alive = false;
        return false;
      }
      const LfCtx &C = ctxs[par];
      if (C.idx < 0) return false;
      gitem = C.gitem;
      T = C.T;
      nbw = C.nbw;
      u_lo = C.u_lo;
      cnt = C.cnt;
      tk0 = C.tk0;
      ng = C.ng;
      dd = C.d;
      direct = C.direct;
      const int code = C.code[q];
      e_lo = C.elo[q];
      e_hi = C.ehi[q];
      active = gitem ? code == 2 : code == 1;
      tO = tmem + lane_off + LF_TM_O(grp, par);
      m_ref = -INFINITY;
      l = 0.f;
      has_pv = false;
      return true;
    };
    // move (k, t) onto the group's next own tile; false at the end
    int t = 0;
    auto settle = [&]() -> bool {
      while (t >= T) {
        t -= T;
        if (!leave()) {
          alive = false;
          return false;
        }
        if (!enter()) return false;
      }
      return true;
    };
    uint32_t x0[32], x1[32];
    // wait for S of own tile c and issue its TMEM loads
    auto fetch = [&](int c) -> bool {
      // The two groups run equal work per tile; started together they stay
      // in step and their non-exp phases coincide.  Group 1 therefore starts
      // its first tile half a tile after group 0 (which arrives on the
      // stagger barrier between its two chunks); the offset persists.
      if (grp == 1 && c == 0 && !lf_wait_warp(BAR(LB_STAGGER), 0, abort_flag, status, 25))
        return false;
      if (!lf_wait_warp(BAR(LB_S_FULL(grp, c & 1)), (c >> 1) & 1, abort_flag, status, 8))
        return false;
      lf_tc_fence_after();
      const uint32_t tS = tmem + lane_off + LF_TM_S(grp, c & 1);
      lf_tmem_ld32_nowait(tS, x0);
      lf_tmem_ld32_nowait(tS + 32, x1);
      return true;
    };
    bool have = enter();
    if (have) {
      t = ((gt & 1) == grp) ? 0 : 1;
      have = settle();
    }
    if (have && !fetch((gt + t) >> 1)) {
      alive = false;
      have = false;
    }
    while (have) {
      const int j = gt + t, c = j >> 1, sb = c & 1;
      const uint32_t tS = tmem + lane_off + LF_TM_S(grp, sb);
      // ---- attend mask of row q over the tile's 64 columns (2 words)
      uint32_t wb[2];
      if (t < nbw) {
        const int kb = tk0 + t * LF_FK;
        int lo = 0, hi = LF_FK - 1;
        if (!gitem) lf_f_band_cols(q, u_lo + t, rr, causal, lo, hi);
        lo = max(lo, -kb);  // keys exist on [0, cnt)
        hi = min(hi, cnt - 1 - kb);
        if (!active) hi = -1;
#pragma unroll
        for (int cc = 0; cc < 2; cc++) {
          uint32_t v;
          if (!direct) {
            v = ctxs[par].vw[2 * t + cc];
          } else {
            const LfCtx &C = ctxs[par];
            const int tk = kb + 32 * cc + lane;
            const int32_t *mrow = D.mask + (size_t)C.b * n;
            v = __ballot_sync(0xffffffffu, tk >= 0 && tk < cnt && mrow[C.rho + tk * dd] != 0);
          }
          wb[cc] = lf_range_bits(lo, hi, 32 * cc) & v;
        }
      } else {
        const LfCtx &C = ctxs[par];
        const int gti = t - nbw, gbs = gti * LF_FK;
        const int hi = active ? min(LF_FK - 1, ng - 1 - gbs) : -1;
#pragma unroll
        for (int cc = 0; cc < 2; cc++) {
          uint32_t inwin = lf_range_bits(e_lo - gbs, e_hi - 1 - gbs, 32 * cc);
          if (dd > 1) {
            uint32_t res;
            if (!direct) {
              res = C.vw[C.rw0 + 2 * gti + cc];
            } else {
              const int e = gbs + 32 * cc + lane;
              const int32_t *gl = D.gidx + (size_t)C.b * D.G;
              res = __ballot_sync(0xffffffffu, e < ng && (gl[e] - C.rho) % dd == 0);
            }
            inwin &= res;
          }
          wb[cc] = lf_range_bits(0, hi, 32 * cc) & ~inwin;
        }
      }
      const bool anyc[2] = {__any_sync(0xffffffffu, wb[0] != 0u) != 0,
                            __any_sync(0xffffffffu, wb[1] != 0u) != 0};
      // ---- the tile's raw scores (loaded ahead), masked, and their max
      lf_tmem_wait_ld_regs(x0);
      lf_tmem_pin_regs(x1);
      float mt = -INFINITY;
      if (anyc[0]) mt = lf_mask_max(x0, wb[0]);
      if (anyc[1]) mt = fmaxf(mt, lf_mask_max(x1, wb[1]));
      mt *= sl2;
      // ---- the row's reference m_ref follows its running max, moved only
      // when a tile's max exceeds it by more than 2^8: then p <= 2^8, so P
      // keeps full precision in bf16 and f16, and a tile's row sum stays far
      // inside every format's range.  Moving it rescales l and the O the
      // group accumulated for this item (after its previous P.V).
      const bool grow = mt > m_ref + 8.f;
      if (__any_sync(0xffffffffu, grow)) {
        const float m_new = grow ? mt : m_ref;
        const float alpha = grow ? lf_ex2(m_ref - m_new) : 1.f;  // 0 when m_ref = -inf
        l *= alpha;
        m_ref = m_new;
        if (has_pv) {
          if (!lf_wait_warp(BAR(LB_PV_DONE(grp)), (c - 1) & 1, abort_flag, status, 10)) {
            alive = false;
            break;
          }
          lf_tc_fence_after();
          lf_rescale_o(tO, alpha);
        }
      }
      // ---- probabilities -> P over the tile's first 32 S columns (the raw
      // scores are in registers already)
      const float mneg = m_ref == -INFINITY ? 0.f : -m_ref;
      float s0 = 0.f, s1 = 0.f;
      lf_p_chunk<kF16>(x0, anyc[0], sl2, mneg, tS, s0, s1);
      if (grp == 0 && c == 0) {
        __syncwarp();
        if (lane == 0) lf_mbar_arrive(BAR(LB_STAGGER));
      }
      lf_p_chunk<kF16>(x1, anyc[1], sl2, mneg, tS + 16, s0, s1);
      l += s0 + s1;
      has_pv = true;
      lf_tmem_wait_st();
      lf_tc_fence_before();
      __syncwarp();
      if (lane == 0) lf_mbar_arrive(BAR(LB_P_FULL(grp, sb)));
      // ---- next own tile: its scores' loads go out now
      t += 2;
      if (!settle()) {
        have = false;
        break;
      }
      if (!fetch((gt + t) >> 1)) {
        alive = false;
        break;
      }
    }
    if (alive && k >= 0 && !have) {
      // (the loop ended on the end marker: nothing left to hand over)
    }
    (void)alive;
  } else {
    // ================================================== epilogue (warps 8-11)
    const int quarter = warp & 3;
    const int q = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    int epi_ph = 0;
    // epilogue-warp barrier (bounded)
    auto epi_sync = [&]() -> bool {
      __syncwarp();
      if (lane == 0) lf_mbar_arrive(BAR(LB_EPI));
      const bool okw = lf_wait_warp(BAR(LB_EPI), epi_ph & 1, abort_flag, status, 21);
      epi_ph++;
      return okw;
    };
    for (int k = 0;; k++) {
      const int par = k & 1;
      if (!lf_wait_warp(BAR(LB_CTX_FULL(par)), (k >> 1) & 1, abort_flag, status, 22)) break;
      const LfCtx &C = ctxs[par];
      if (C.idx < 0) break;
      const int gitem = C.gitem, b = C.b, h = C.h, qrow0 = C.qrow0, kt0 = C.kt0;
      const int code = C.code[q], pos = C.pos[q];
      __syncwarp();
      if (lane == 0) lf_mbar_arrive(BAR(LB_CTX_EMPTY(par)));
      if (!lf_wait_warp(BAR(LB_ML_FULL(par)), (k >> 1) & 1, abort_flag, status, 23)) break;
      const float2 mla = mls[(par * 2 + 0) * 128 + q], mlb = mls[(par * 2 + 1) * 128 + q];
      __syncwarp();
      if (lane == 0) lf_mbar_arrive(BAR(LB_ML_EMPTY(par)));
      if (!lf_wait_warp(BAR(LB_O_FULL(par)), (k >> 1) & 1, abort_flag, status, 24)) break;
      lf_tc_fence_after();
      const uint32_t tOa = tmem + lane_off + LF_TM_O(0, par), tOb = tmem + lane_off + LF_TM_O(1, par);
      // merge the groups: a group with nothing summed contributes nothing
      // (its O columns may hold another item's values)
      const float m = fmaxf(mla.y > 0.f ? mla.x : -INFINITY, mlb.y > 0.f ? mlb.x : -INFINITY);
      const float fa = mla.y > 0.f ? lf_ex2(mla.x - m) : 0.f;
      const float fb = mlb.y > 0.f ? lf_ex2(mlb.x - m) : 0.f;
      const float L = fa * mla.y + fb * mlb.y;
      const size_t bh = (size_t)b * D.H + h;
      const bool store_band = !gitem && code >= 0 && code != 2;
      const bool store_g = gitem && code == 2;
      const float inv = (code == 1 && L > 0.f) ? 1.f / L : 0.f;
      const size_t pi =
          gitem ? ((bh * D.G + (qrow0 + q)) * D.nch + kt0 / (D.chunk_tiles * (LF_BK / LF_FK))) : 0;
      const size_t orow = bh * n + pos;
      // O of both groups: the row is merged and stored half by half (O is
      // double-buffered by item parity, so it is freed for the item two
      // ahead after the second half's loads without delaying anything)
#pragma unroll
      for (int half = 0; half < 2; half++) {
        uint32_t ra[32], rb[32];
        lf_tmem_ld32_nowait(tOa + 32 * half, ra);
        lf_tmem_ld32_nowait(tOb + 32 * half, rb);
        lf_tmem_wait_ld_regs(ra);
        lf_tmem_pin_regs(rb);
        if (half == 1) {
          lf_tc_fence_before();
          __syncwarp();
          if (lane == 0) lf_mbar_arrive(BAR(LB_O_FREE(par)));
        }
#pragma unroll
        for (int kk = 0; kk < 32; kk++) {
          const float a = fa > 0.f ? fa * __uint_as_float(ra[kk]) : 0.f;
          const float bb = fb > 0.f ? fb * __uint_as_float(rb[kk]) : 0.f;
          ra[kk] = __float_as_uint(a + bb);
        }
        if (store_band) {
          uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<uint16_t *>(P.o) + orow * LF_HD) +
                       4 * half;
#pragma unroll
          for (int kk = 0; kk < 4; kk++) {
            uint4 u;
            u.x = lf_pack2<kF16>(__uint_as_float(ra[8 * kk + 0]) * inv, __uint_as_float(ra[8 * kk + 1]) * inv);
            u.y = lf_pack2<kF16>(__uint_as_float(ra[8 * kk + 2]) * inv, __uint_as_float(ra[8 * kk + 3]) * inv);
            u.z = lf_pack2<kF16>(__uint_as_float(ra[8 * kk + 4]) * inv, __uint_as_float(ra[8 * kk + 5]) * inv);
            u.w = lf_pack2<kF16>(__uint_as_float(ra[8 * kk + 6]) * inv, __uint_as_float(ra[8 * kk + 7]) * inv);
            dst[kk] = u;
          }
        } else if (store_g) {
          float4 *dst = reinterpret_cast<float4 *>(P.part_acc + pi * LF_HD) + 8 * half;
#pragma unroll
          for (int kk = 0; kk < 8; kk++)
            dst[kk] = make_float4(__uint_as_float(ra[4 * kk]), __uint_as_float(ra[4 * kk + 1]),
                                  __uint_as_float(ra[4 * kk + 2]), __uint_as_float(ra[4 * kk + 3]));
        }
      }
      if (store_band && P.lse) P.lse[orow] = code == 1 ? (m + __log2f(L)) * LF_LN2 : -INFINITY;
      if (gitem) {
        // split-KV partial of the global row; the CTA that completes a row
        // group's partials merges them into O and lse
        if (store_g) P.part_ml[pi] = make_float2(m, L);
        __threadfence();
        if (!epi_sync()) break;
        if (q == 0) {
          const int qt = qrow0 / LF_BQ;
          const int old = atomicAdd(P.gcount + (bh * P.ngq + qt), 1);
          *epi_flag = old == D.nch - 1 ? 1 : 0;
        }
        if (!epi_sync()) break;
        const bool last = *epi_flag != 0;
        if (last && store_g) {
          __threadfence();
          const size_t base = (bh * D.G + (qrow0 + q)) * D.nch;
          float mm = -INFINITY;
          for (int ch = 0; ch < D.nch; ch++) mm = fmaxf(mm, __ldcg(&P.part_ml[base + ch]).x);
          float LL = 0.f;
          uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<uint16_t *>(P.o) + orow * LF_HD);
          // two halves of 32 columns (keeps the accumulator small)
#pragma unroll 1
          for (int half = 0; half < 2; half++) {
            float acc[32];
#pragma unroll
            for (int kk = 0; kk < 32; kk++) acc[kk] = 0.f;
            float lsum = 0.f;
            for (int ch = 0; ch < D.nch; ch++) {
              const float2 ml = __ldcg(&P.part_ml[base + ch]);
              if (ml.y == 0.f) continue;
              const float f = lf_ex2(ml.x - mm);
              lsum += ml.y * f;
              const float4 *src =
                  reinterpret_cast<const float4 *>(P.part_acc + (base + ch) * LF_HD) + 8 * half;
#pragma unroll
              for (int kk = 0; kk < 8; kk++) {
                const float4 av = __ldcg(src + kk);
                acc[4 * kk] += av.x * f;
                acc[4 * kk + 1] += av.y * f;
                acc[4 * kk + 2] += av.z * f;
                acc[4 * kk + 3] += av.w * f;
              }
            }
            LL = lsum;
            const float il = lsum > 0.f ? 1.f / lsum : 0.f;
#pragma unroll
            for (int kk = 0; kk < 4; kk++) {
              uint4 u;
              u.x = lf_pack2<kF16>(acc[8 * kk + 0] * il, acc[8 * kk + 1] * il);
              u.y = lf_pack2<kF16>(acc[8 * kk + 2] * il, acc[8 * kk + 3] * il);
              u.z = lf_pack2<kF16>(acc[8 * kk + 4] * il, acc[8 * kk + 5] * il);
              u.w = lf_pack2<kF16>(acc[8 * kk + 6] * il, acc[8 * kk + 7] * il);
              dst[4 * half + kk] = u;
            }
          }
          if (P.lse) P.lse[orow] = (mm + __log2f(LL)) * LF_LN2;
        }
      }
    }
  }

  // ---------------------------------------------------- teardown
  lf_tc_fence_before();
  __syncthreads();
  if (warp == 13) {
    lf_tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(LF_TM_COLS)
                 : "memory");
  }
}
// ------------------------------------------------------------ gather (backward)

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
                 uint64_t B, uint64_t row_stride, uint64_t head_stride, uint64_t batch_stride,
                 uint32_t box_rows) {
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

// 2-D map over all rows [rows, 64] with a one-row box: the source of the
// four-row TMA gathers (128-byte swizzle, like the tiled maps).
static bool lf_make_gather_map(CUtensorMap *m, int f16, const void *base, uint64_t rows) {
  PFN_cuTensorMapEncodeTiled enc = lf_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {64, rows};
  cuuint64_t strides[1] = {128};
  cuuint32_t box[2] = {64, 1};
  cuuint32_t es[2] = {1, 1};
  CUresult r = enc(m, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
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
static cudaError_t lf_launch_pdl(const void *fn, unsigned grid, unsigned block, size_t smem,
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

// Parameter block staging (host): too large for the stack of every caller.
static thread_local LfFwdParams g_fwd_params;

int lf_tc_fwd(const LfLaunch &L, const LfTcArgs &a, char *err, size_t errlen) {
  const LfDev &D = L.dev;
  const int f16 = L.dtype == LF_F16 ? 1 : 0;
  LfFwdParams &P = g_fwd_params;  // the launch copies the parameter block
  memset(&P, 0, sizeof(P));
  P.dev = D;
  const uint64_t n = D.n, H = D.H, B = D.B, rowb = 128;
  int nmaps = 0;
  // segments: runs of heads with equal dilation x residues; each residue view
  // (d, rho) has three maps (Q_s, K_s, V_s) with row stride d rows
  std::map<std::pair<int, int>, int> rmap;
  int nseg = 0, start1 = 0, start2 = 0;
  const int el = (D.r + LF_BQ - 1) / LF_BQ;          // edge blocks at the start
  const int er = D.causal ? 0 : (D.r + LF_BQ - 1) / LF_BQ;  // and at the end
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
        if (nmaps + 3 > LF_F_MAX_MAPS - 5) {
          snprintf(err, errlen,
                   "tensor-core path: too many distinct dilation residues (the sum of the distinct "
                   "dilations must stay <= %d)", (LF_F_MAX_MAPS - 5) / 3);
          return LF_ERR_UNSUPPORTED;
        }
        // Q: 128-row box (a block of queries); K, V: 64-row box (a key tile)
        const char *srcs[3] = {(const char *)a.qs, (const char *)a.ks, (const char *)a.vs};
        for (int k = 0; k < 3; k++)
          if (!lf_make_map(&P.maps[nmaps + k], f16, srcs[k] + rho * rowb, cnt, H, B, d * rowb,
                           n * rowb, H * n * rowb, k == 0 ? LF_BQ : LF_FK)) {
            snprintf(err, errlen, "tensor map encode failed (d=%d, rho=%d)", d, rho);
            return LF_ERR_CUDA;
          }
        rmap[key] = nmaps;
        nmaps += 3;
      }
      if (nseg >= LF_F_MAX_SEG) {
        snprintf(err, errlen, "tensor-core path: too many (dilation run, residue) segments (> %d)",
                 LF_F_MAX_SEG);
        return LF_ERR_UNSUPPORTED;
      }
      const int nl = std::min(el, nqb), nr = std::min(er, nqb - nl);
      P.seg[nseg] = LfFSeg{h0, h1, d, rho, cnt, nqb, nl, nr, start1, start2, rmap[key]};
      start1 += (h1 - h0) * (nqb - nl - nr);
      start2 += (h1 - h0) * (nl + nr);
      nseg++;
    }
    h0 = h1;
  }
  P.nseg = nseg;
  P.per1 = start1;
  P.per2 = start2;
  // global rows: K_g / V_g tiled maps; gather maps over every row of Q_g,
  // K_s, V_s
  const int G = D.G;
  P.map_kg = nmaps;
  P.map_vg = nmaps + 1;
  P.map_qg2 = nmaps + 2;
  P.map_ks2 = nmaps + 3;
  P.map_vs2 = nmaps + 4;
  const uint64_t allrows = B * H * n;
  bool ok = lf_make_map(&P.maps[nmaps], f16, a.kg, n, H, B, rowb, n * rowb, H * n * rowb, LF_FK) &&
            lf_make_map(&P.maps[nmaps + 1], f16, a.vg, n, H, B, rowb, n * rowb, H * n * rowb, LF_FK) &&
            lf_make_gather_map(&P.maps[nmaps + 2], f16, a.qg, allrows) &&
            lf_make_gather_map(&P.maps[nmaps + 3], f16, a.ks, allrows) &&
            lf_make_gather_map(&P.maps[nmaps + 4], f16, a.vs, allrows);
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
  P.gcount = (int *)(L.ws_base + L.ws.status) + LF_ST_WORDS;
  // the mask pass: global list, rank array, sequence info, input checks
  cudaError_t e = lf_launch_mask_pass(L);
  if (e != cudaSuccess) {
    snprintf(err, errlen, "mask pass launch: %s", cudaGetErrorString(e));
    return LF_ERR_CUDA;
  }
  void (*kern)(const LfFwdParams) = f16 ? lf_tc_fwd_kernel<1> : lf_tc_fwd_kernel<0>;
  e = lf_kernel_smem((const void *)kern, LF_SMEM_BYTES);
  if (e != cudaSuccess) {
    snprintf(err, errlen, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    return LF_ERR_CUDA;
  }
  const long long items = (long long)P.n_gitems + (long long)D.B * (P.per1 + P.per2);
  const unsigned grid = (unsigned)std::max<long long>(1, std::min<long long>(items, lf_sm_count()));
  if (a.ev_start && a.ev_stop) cudaEventRecord(a.ev_start, L.stream);
  void *args[] = {(void *)&P};
  cudaError_t le = lf_launch_pdl((const void *)kern, grid, LF_F_THREADS, LF_SMEM_BYTES, L.stream, args);
  lf_launches_add(1);
  if (a.ev_start && a.ev_stop) cudaEventRecord(a.ev_stop, L.stream);
  e = le != cudaSuccess ? le : cudaGetLastError();
  if (e != cudaSuccess) {
    snprintf(err, errlen, "tensor-core forward launch: %s", cudaGetErrorString(e));
    return LF_ERR_CUDA;
  }
  return LF_OK;
}

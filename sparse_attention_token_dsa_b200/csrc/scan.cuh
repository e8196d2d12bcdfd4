// scan.cuh — the indexer scan: tcgen05 scoring tile + fused ReLU / head-weight
// reduction / causal mask + streaming exact top-k filter.
//
// Computes, for every query row t of a work item and every legal key s,
//     I_{t,s} = sum_j w_{t,j} * ReLU(q_{t,j} . k_s)          (DSA indexer score)
// ("PaperTrace 2.2.2 MISA, LISA and ResMiSA", opening DSA definition; the
// kernel fuses score, causal mask and top-k so the n^2 score matrix never
// reaches memory, section 2.2 "kernel boundary").  Restricted to a routed
// head subset this is MISA's step 4 ("MISA: Mixture of Indexer Sparse
// Attention", method step 4): the caller passes gathered q / w rows.  The
// keys of a work item are a contiguous range, full-block representatives
// (HISA's coarse stage), or a per-row list gathered by TMA (the MISA-dagger and
// HISA reranks, whose rows select once at the end instead of streaming).
//
// Layout of one CTA (persistent, one per SM, one work item at a time):
//   warps 0-7  epilogue: TMEM -> registers, ReLU, * w, sum over heads, causal
//              mask, composite key, threshold filter, append to warp-owned
//              candidate sub-logs, per-row threshold maintenance
//   warp 8     TMA producer: Q tile of the item (resident), K tiles streamed
//              through 2-6 stages
//   warp 9     MMA issuer (one thread) + TMEM allocator
// MMA: M = 128 keys (TMEM lane = key), N = query rows x heads, K = d (the
// split-query fp8 form issues its hi and lo query parts as two MMAs into the
// same accumulator); fp32 accumulate in TMEM, 2-8 accumulator stages so the
// epilogue of one unit overlaps the MMAs of the next.
//
// Streaming top-k.  A candidate (score, key) is kept while its composite key
// (order-preserving score bits, then ~index) is >= the row's threshold thr.
// thr is always a lower bound of the row's final keep-th best composite, so no
// winner is ever dropped.  It is raised every kUpdateSteps steps from per-row
// histograms of the kept candidates: h1 counts them by the top byte of the
// 32-bit score key; h2[0] / h2[1] count those whose top byte equals b1 / b1 + 1
// by the second byte, where b1 is the top-byte bin holding the keep-th best.
// The pair gives thr at 16-bit score-key resolution (bf16 precision) without
// rescanning the logs; a first threshold, or a jump of b1 by more than one,
// restarts h2 empty (thr then has top-byte resolution until h2 has counted
// enough new candidates).  Counts can only be low (never high) in the bins the
// search reaches, which can only make thr looser, never invalid.  Each epilogue warp
// appends to its own sub-log per row (no atomics) and compacts it in place
// (keep >= thr) when it nears capacity; if that is not enough (long runs of
// tied scores) an exact radix-select raise sets thr to the keep-th best
// composite itself.
#pragma once
#include "common.cuh"
#include "select.cuh"

namespace dsa {

struct ScanArgs {
  int32_t batch, n_q, n_k, H, d;
  int32_t q_stride;      // query rows per sequence in q / w / scales (>= q_off + n_q)
  int32_t q_off;         // first query of this call: row i of sequence b is q / w row
                         //   b * q_stride + q_off + i, at position pos0 + q_off + i
  int32_t n_tok;         // token positions per sequence (default pos0 = n_tok - q_stride,
                         //   k_len = n_tok)
  int32_t bs_shift;      // > 0: keys are full-block representatives of 2^bs_shift tokens;
                         //      a row sees block b iff (b + 1) << bs_shift <= min(pos + 1, k_len)
  const int32_t* klist;  // gathered keys: per-row lists [rows, klist_len] (-1 = empty slot)
  int32_t klist_len;
  const uint16_t* kraw;  // token-list gathers: the key rows themselves [batch * n_k, 128] bf16
  int32_t lb_shift;      // block lists: log2 tokens per listed block
  int32_t keep;          // entries each row must keep (top-k or k')
  int32_t QG;            // query rows per accumulator group (<= 256 / (H * parts))
  int32_t qcols;         // Q-tile rows per group: max(16, QG * H) x parts; MMA N = qcols / parts
  int32_t G;             // groups per work item (1 or 2)
  int32_t stage_cols;    // TMEM columns per accumulator stage (64, 128 or 256)
  int32_t tstages;       // accumulator stages in TMEM (2 .. 8; tstages * stage_cols <= 512)
  int32_t kstages;       // K-stage pipeline depth (2 .. 6)
  int32_t kt;            // 128-key tiles per K stage and accumulator unit (1 or 2; 2 only
                         // with one query row per item, G = QG = 1)
  int32_t n_qt;          // query tiles per sequence (ceil(n_q / (QG*G)))
  int32_t C;             // key chunks per row (split-K); 1 = whole prefix
  int32_t chunk;         // keys per chunk (multiple of 128) when C > 1
  int32_t n_items;       // batch * n_qt * C
  const int32_t* q_pos0; // [batch] or null: n_tok - q_stride
  const int32_t* k_len;  // [batch] or null: n_k
  const float* w;        // [rows, H]
  const float* row_scale;   // [rows] or null: multiplies w (query dequant scale)
  const float* head_scale;  // [rows, H] or null: multiplies w (split-query scale)
  const float* k_scale;     // [batch * n_k] or null: multiplies the score (key dequant scale)
  int32_t nsub;          // sub-logs per row slot (4: one per lane quadrant; 8: one per warp)
  int32_t capw;          // entries per sub-log (>= keep + 256)
  uint64_t* logs;        // [rows * C][nsub][capw] composite keys
  int32_t* log_cnt;      // [rows * C][nsub]
  unsigned long long* log_thr;  // [rows * C] final threshold of the slot
  int32_t* status;       // workspace status word
  long long wait_cycles; // budget of every bounded wait (kWaitCycles; shorter in tests)
  const float* dosa_ub;  // DoSA: per (row, block) upper bounds of I [rows, dosa_nblk], or null
  int32_t dosa_nblk;     //   bound blocks per row
  int32_t dosa_shift;    //   log2 tokens per bound block (>= 7: a key tile lies in one block)
  unsigned long long* dosa_pruned;  // (row, unit) pairs skipped, or null
  const float* dosa_seed;  // DoSA: per row a lower bound of its keep-th best score [rows]
                           //   (-inf: none), the row threshold's starting value
  const unsigned long long* dosa_counts;  // DoSA: (row, block) pairs with legal keys, and
                           //   those the seeds alone rule out; the block checks run only
                           //   when at least 1/32 of them are
  int32_t test_stall;    // DSA_FLAG_TEST_STALL: CTA 0 withholds the second K stage of
                         //   its first item, so the waits on it run out (tests only)
};

constexpr int kEpiWarps = 8;
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kScanThreads = 320;
constexpr int kMaxRows = 16;          // rows per work item
constexpr int kMaxItemCols = 512;     // rows x heads per item
constexpr int kBarEpi = 1;            // named barrier among the epilogue warps
constexpr int kHistWords = 768;       // h1[256] + h2[2][256] per row
constexpr int kUpdateSteps = 16;      // steps (key tiles) between threshold updates
// Sub-log slack: a step appends at most 64 entries per row to one sub-log, and a
// flagged row waits at most two update periods for its exact raise.
constexpr int kCompactSlack = 64 * 2 * kUpdateSteps + 128;
// Gathered-key rows keep every candidate of their list in shared memory and
// select once at the end of the row.
constexpr int kMaxGatherKeys = 8192;
constexpr int kGatherBins = 4096;     // linear score bins of the end-of-row selection
constexpr int kGatherBoundary = 256;  // boundary-bin candidates ranked by one warp
constexpr int kMaxTStages = 8;

template <MmaKind KIND>
struct ScanCfg {
  static constexpr int ESZ = KIND == MmaKind::TF32 ? 4 : (KIND == MmaKind::BF16 ? 2 : 1);
  static constexpr int A = 128 * ESZ / 128;   // 128-byte atoms per key row (d = 128)
  static constexpr int EPA = 128 / ESZ;       // elements per atom
  static constexpr int KTILE_BYTES = A * 128 * 128;
};

struct ScanSmemTail {
  uint64_t k_full[8], k_empty[8];
  uint64_t q_full, q_empty;
  uint64_t t_full[kMaxTStages], t_empty[kMaxTStages];
  uint64_t drain;
  uint32_t tmem_base;
  int32_t abort;
  int32_t epi_stop[2];
  int32_t raise_snap[2];
  int32_t row_nleg[kMaxRows];  // legal keys of the row in this item, counted from kbeg
  int32_t row_b1[kMaxRows];    // top-byte bin of the keep-th best (-1: fewer kept)
  int32_t row_raise[kMaxRows]; // a sub-log could not be compacted enough
  int32_t raise_any;           // some row needs an exact raise
  int32_t gather_legal;        // gathered row: legal candidates seen
  int32_t gather_nwin, gather_nbnd;
  float gather_lo[kEpiWarps], gather_hi[kEpiWarps];
  int32_t subcnt[kMaxRows][8]; // sub-log fill, written only by the owning warp
  unsigned long long row_thr[kMaxRows];
  int32_t item_min_nleg;       // smallest row_nleg of the item's rows
  unsigned int dosa_skips;     // (row, unit) pairs this CTA skipped by their DoSA bound
  alignas(16) float wsm[kMaxItemCols];
  SelectScratch sel;
};

struct ItemGeom {
  int b, qt, c, row0, nrows, kbeg, kend, ntiles, t_hi;
};

template <int GATHER>
__device__ __forceinline__ ItemGeom item_geom(const ScanArgs& a, int item) {
  ItemGeom g;
  const int qt_rev = item / (a.batch * a.C);
  const int rem = item % (a.batch * a.C);
  g.b = rem / a.C;
  g.c = rem % a.C;
  g.qt = a.n_qt - 1 - qt_rev;
  const int QT = a.QG * a.G;
  g.row0 = g.qt * QT;
  g.nrows = min(QT, a.n_q - g.row0);
  if constexpr (GATHER != 0) {
    // one row per item; its keys come from its list, in list order (a block
    // list expands each entry into 2^lb_shift consecutive tokens)
    const int nkeys = GATHER == 2 ? (a.klist_len << a.lb_shift) : a.klist_len;
    g.kbeg = 0;
    g.kend = nkeys;
    g.ntiles = g.nrows > 0 ? (nkeys + 127) >> 7 : 0;
    g.t_hi = 0;
    return g;
  }
  const int pos0 = (a.q_pos0 ? a.q_pos0[g.b] : a.n_tok - a.q_stride) + a.q_off;
  const int klen = a.k_len ? a.k_len[g.b] : a.n_tok;
  const int maxpos = pos0 + g.row0 + g.nrows - 1;
  int kend = min(maxpos + 1, klen);
  if (a.bs_shift > 0) kend = kend >> a.bs_shift;  // full blocks only
  int kbeg = 0;
  if (a.C > 1) {
    kbeg = g.c * a.chunk;
    kend = min(kend, kbeg + a.chunk);
  }
  g.kbeg = kbeg;
  g.kend = kend;
  if (g.nrows <= 0 || kend <= kbeg) {
    g.ntiles = 0;
    g.t_hi = 0;
  } else {
    g.t_hi = (kend - 1) >> 7;
    g.ntiles = g.t_hi - (kbeg >> 7) + 1;
  }
  return g;
}

// Snake-ordered static schedule: items are ordered longest-first; CTA c takes
// item c of round 0, item G-1-c of round 1, ... so causal lengths balance.
__device__ __forceinline__ int sched_item(int round, int cta, int grid) {
  return round * grid + ((round & 1) ? (grid - 1 - cta) : cta);
}

// In-place warp compaction of one sub-log: keep entries >= thr; returns the
// count.  Rounds of 256 entries (eight loads per lane); the next round's loads
// are issued before this round's writes, which land below the next round's
// range (the write position never passes the read position), so they overlap.
__device__ __forceinline__ int compact_sublog(uint64_t* lg, int n, unsigned long long thr,
                                              int lane) {
  int wpos = 0;
  uint64_t cur[8], nxt[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int i = j * 32 + lane;
    cur[j] = i < n ? lg[i] : 0ull;
  }
  for (int i0 = 0; i0 < n; i0 += 256) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int i = i0 + 256 + j * 32 + lane;
      nxt[j] = i < n ? lg[i] : 0ull;
    }
    __syncwarp();
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int i = i0 + j * 32 + lane;
      const bool kp = i < n && cur[j] >= thr;
      const unsigned bal = __ballot_sync(0xffffffffu, kp);
      if (kp) lg[wpos + __popc(bal & ((1u << lane) - 1))] = cur[j];
      wpos += __popc(bal);
    }
    __syncwarp();
#pragma unroll
    for (int j = 0; j < 8; ++j) cur[j] = nxt[j];
  }
  return wpos;
}

// Per-unit context of the filter: the lane's key, its dequant scale, and where
// this warp's sub-logs and the row histograms live.
struct FilterCtx {
  int key;
  float ks;
  int kbeg;
  int lane;
  unsigned lanemask_lt;
  int sub;
  bool all_legal;        // every key of this unit is legal for every row of the item
  uint64_t* logs;        // this warp's sub-log of item row 0
  uint32_t row_stride;   // entries between consecutive rows' sub-logs
  uint32_t* hist;
  ScanSmemTail* T;
  int capw;              // sub-log capacity (a write past it is recorded, not made)
  int32_t* status;
};

// Legality, composite key, threshold filter and append for one query row.
// The common path (no lane survives) costs the key arithmetic, one threshold
// load and a vote (the legality test is skipped for units inside every row's
// legal range).
// the key arithmetic and a vote.
__device__ __forceinline__ void filter_append(const FilterCtx& f, int r, float acc) {
  ScanSmemTail* T = f.T;
  const bool legal = f.all_legal || (unsigned)(f.key - f.kbeg) < (unsigned)T->row_nleg[r];
  const uint32_t sk = score_key(acc * f.ks);
  const uint64_t comp = ((uint64_t)sk << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)f.key);
  const bool surv = legal && comp >= T->row_thr[r];
  const unsigned bal = __ballot_sync(0xffffffffu, surv);
  if (bal) {
    int* cnt = &T->subcnt[r][f.sub];
    const int base = *cnt;
    if (base + __popc(bal) > f.capw) {
      // cannot happen while compaction keeps its slack; never write past the log
      if (f.lane == 0) set_status(f.status, DSA_ERR_INTERNAL, 110);
      return;
    }
    if (surv) {
      f.logs[(uint32_t)r * f.row_stride + (uint32_t)(base + __popc(bal & f.lanemask_lt))] = comp;
      uint32_t* h = f.hist + r * kHistWords;
      const int b1 = (int)(sk >> 24);
      atomicAdd(&h[b1], 1u);
      const unsigned d1 = (unsigned)(b1 - T->row_b1[r]);
      if (d1 <= 1u) atomicAdd(&h[256 + d1 * 256 + ((sk >> 16) & 255)], 1u);
    }
    __syncwarp();
    if (f.lane == 0) *cnt = base + __popc(bal);
    __syncwarp();
  }
}

// Packed fp32 pair FMA (sm_100a): acc.{x,y} += w.{x,y} * {a, b}, each lane an
// IEEE round-to-nearest fma, identical to two scalar fmaf.
__device__ __forceinline__ void ffma2(unsigned long long& acc, unsigned long long w, float a,
                                      float b) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(w), "l"(r));
}
__device__ __forceinline__ float pair_sum(unsigned long long v) {
  float a, b;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
  return a + b;
}

// sum_j w_j ReLU(v_j) over NC 32-column chunks into four packed partial sums.
template <int NC>
__device__ __forceinline__ void relu_dot(const uint32_t (&v)[NC][32], const float* w,
                                         unsigned long long (&acc)[4]) {
#pragma unroll
  for (int c = 0; c < NC; ++c) {
#pragma unroll
    for (int jj = 0; jj < 32; jj += 4) {
      const ulonglong2 wv = *reinterpret_cast<const ulonglong2*>(w + c * 32 + jj);
      const int o = (jj >> 2) & 1;
      ffma2(acc[2 * o + 0], wv.x, fmaxf(__uint_as_float(v[c][jj + 0]), 0.f),
            fmaxf(__uint_as_float(v[c][jj + 1]), 0.f));
      ffma2(acc[2 * o + 1], wv.y, fmaxf(__uint_as_float(v[c][jj + 2]), 0.f),
            fmaxf(__uint_as_float(v[c][jj + 3]), 0.f));
    }
  }
}

template <int NC>
__device__ __forceinline__ void tmem_ld_chunks(uint32_t taddr, uint32_t (&v)[NC][32]) {
#pragma unroll
  for (int c = 0; c < NC; ++c) tmem_ld32(taddr + c * 32, v[c]);
}
template <int NC>
__device__ __forceinline__ void tmem_wait_chunks(uint32_t (&v)[NC][32]) {
#pragma unroll
  for (int c = 0; c < NC; ++c) tmem_ld_wait(v[c]);
}

__device__ __forceinline__ float sum8(const unsigned long long (&a)[4]) {
  return (pair_sum(a[0]) + pair_sum(a[1])) + (pair_sum(a[2]) + pair_sum(a[3]));
}

// One unit of this warp: nq query rows of HT heads starting at TMEM column
// address `col` (row r = rbase + i, weights w + i * HT).  Work is split into
// segments of at most 64 columns; the TMEM loads of segment i+1 are in flight
// while segment i is reduced.
template <int HT>
__device__ __forceinline__ void unit_heads(const FilterCtx& f, uint32_t col, const float* w,
                                           int nq, int rbase) {
  if constexpr (HT >= 32) {
    constexpr int SEGC = 1;                       // 32-column chunks per segment
    constexpr int SPQ = HT / (32 * SEGC);          // segments per query row
    const int nseg = nq * SPQ;
    uint32_t va[SEGC][32], vb[SEGC][32];
    unsigned long long acc[4] = {0ull, 0ull, 0ull, 0ull};
    tmem_ld_chunks<SEGC>(col, va);
    tmem_wait_chunks<SEGC>(va);
    for (int sg = 0; sg < nseg; sg += 2) {
      const bool has_b = sg + 1 < nseg;
      if (has_b) tmem_ld_chunks<SEGC>(col + (sg + 1) * 32 * SEGC, vb);
      relu_dot<1>(va, w + sg * 32 * SEGC, acc);
      if ((sg + 1) % SPQ == 0) {
        filter_append(f, rbase + sg / SPQ, sum8(acc));
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[i] = 0ull;
      }
      if (!has_b) break;
      tmem_wait_chunks<SEGC>(vb);
      if (sg + 2 < nseg) tmem_ld_chunks<SEGC>(col + (sg + 2) * 32 * SEGC, va);
      relu_dot<1>(vb, w + (sg + 1) * 32 * SEGC, acc);
      if ((sg + 2) % SPQ == 0) {
        filter_append(f, rbase + (sg + 1) / SPQ, sum8(acc));
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[i] = 0ull;
      }
      if (sg + 2 < nseg) tmem_wait_chunks<SEGC>(va);
    }
  } else {
    // HT in {8, 16}: one 32-column chunk holds 32 / HT query rows
    constexpr int QPC = 32 / HT;
    const int nchunk = (nq + QPC - 1) / QPC;
    uint32_t va[1][32], vb[1][32];
    auto chunk = [&](const uint32_t (&v)[1][32], int c) {
#pragma unroll
      for (int qq = 0; qq < QPC; ++qq) {
        if (c * QPC + qq >= nq) break;
        float b[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int jj = 0; jj < HT; jj += 4) {
          const float4 wv = *reinterpret_cast<const float4*>(w + c * 32 + qq * HT + jj);
          b[0] = fmaf(wv.x, fmaxf(__uint_as_float(v[0][qq * HT + jj + 0]), 0.f), b[0]);
          b[1] = fmaf(wv.y, fmaxf(__uint_as_float(v[0][qq * HT + jj + 1]), 0.f), b[1]);
          b[2] = fmaf(wv.z, fmaxf(__uint_as_float(v[0][qq * HT + jj + 2]), 0.f), b[2]);
          b[3] = fmaf(wv.w, fmaxf(__uint_as_float(v[0][qq * HT + jj + 3]), 0.f), b[3]);
        }
        filter_append(f, rbase + c * QPC + qq, (b[0] + b[1]) + (b[2] + b[3]));
      }
    };
    tmem_ld_chunks<1>(col, va);
    tmem_wait_chunks<1>(va);
    for (int c = 0; c < nchunk; c += 2) {
      const bool has_b = c + 1 < nchunk;
      if (has_b) tmem_ld_chunks<1>(col + (c + 1) * 32, vb);
      chunk(va, c);
      if (!has_b) break;
      tmem_wait_chunks<1>(vb);
      if (c + 2 < nchunk) tmem_ld_chunks<1>(col + (c + 2) * 32, va);
      chunk(vb, c + 1);
      if (c + 2 < nchunk) tmem_wait_chunks<1>(va);
    }
  }
}

// unit_heads with the row count known at compile time (HT >= 32): the whole
// unit is one straight-line sequence of 32-column segments, the load of
// segment i+1 in flight while segment i is reduced.
template <int HT, int NQ>
__device__ __forceinline__ void unit_heads_n(const FilterCtx& f, uint32_t col, const float* w,
                                             int rbase) {
  static_assert(HT >= 32, "32-column segments");
  constexpr int SPQ = HT / 32;                 // segments per query row
  constexpr int NSEG = NQ * SPQ;
  uint32_t v[2][1][32];
  unsigned long long acc[4] = {0ull, 0ull, 0ull, 0ull};
  tmem_ld_chunks<1>(col, v[0]);
  tmem_wait_chunks<1>(v[0]);
#pragma unroll
  for (int sg = 0; sg < NSEG; ++sg) {
    if (sg + 1 < NSEG) tmem_ld_chunks<1>(col + (sg + 1) * 32, v[(sg + 1) & 1]);
    relu_dot<1>(v[sg & 1], w + sg * 32, acc);
    if ((sg + 1) % SPQ == 0) {
      filter_append(f, rbase + sg / SPQ, sum8(acc));
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[i] = 0ull;
    }
    if (sg + 1 < NSEG) tmem_wait_chunks<1>(v[(sg + 1) & 1]);
  }
}

// unit_heads for HT in {8, 16} with the row count known at compile time: each
// 32-column chunk holds 32 / HT rows; straight-line, next chunk's load in flight.
template <int HT, int NQ>
__device__ __forceinline__ void unit_heads_small(const FilterCtx& f, uint32_t col, const float* w,
                                                 int rbase) {
  static_assert(HT < 32 && NQ % (32 / HT) == 0, "whole chunks");
  constexpr int QPC = 32 / HT;
  constexpr int NCH = NQ / QPC;
  uint32_t v[2][1][32];
  tmem_ld_chunks<1>(col, v[0]);
  tmem_wait_chunks<1>(v[0]);
#pragma unroll
  for (int c = 0; c < NCH; ++c) {
    if (c + 1 < NCH) tmem_ld_chunks<1>(col + (c + 1) * 32, v[(c + 1) & 1]);
#pragma unroll
    for (int qq = 0; qq < QPC; ++qq) {
      float b[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int jj = 0; jj < HT; jj += 4) {
        const float4 wv = *reinterpret_cast<const float4*>(w + c * 32 + qq * HT + jj);
        b[0] = fmaf(wv.x, fmaxf(__uint_as_float(v[c & 1][0][qq * HT + jj + 0]), 0.f), b[0]);
        b[1] = fmaf(wv.y, fmaxf(__uint_as_float(v[c & 1][0][qq * HT + jj + 1]), 0.f), b[1]);
        b[2] = fmaf(wv.z, fmaxf(__uint_as_float(v[c & 1][0][qq * HT + jj + 2]), 0.f), b[2]);
        b[3] = fmaf(wv.w, fmaxf(__uint_as_float(v[c & 1][0][qq * HT + jj + 3]), 0.f), b[3]);
      }
      filter_append(f, rbase + c * QPC + qq, (b[0] + b[1]) + (b[2] + b[3]));
    }
    if (c + 1 < NCH) tmem_wait_chunks<1>(v[(c + 1) & 1]);
  }
}

// sum_j w_j ReLU(D_j) over the HT accumulator columns of one query row (TMEM
// columns [0, HT) at taddr), for the gathered-key epilogue.
template <int HT>
__device__ __forceinline__ float row_acc(uint32_t taddr, const float* w) {
  if constexpr (HT >= 32) {
    constexpr int NC = HT / 32;
    unsigned long long acc[4] = {0ull, 0ull, 0ull, 0ull};
    uint32_t va[1][32], vb[1][32];
    tmem_ld_chunks<1>(taddr, va);
    tmem_wait_chunks<1>(va);
#pragma unroll
    for (int c = 0; c < NC; c += 2) {
      if (c + 1 < NC) tmem_ld_chunks<1>(taddr + (c + 1) * 32, vb);
      relu_dot<1>(va, w + c * 32, acc);
      if (c + 1 >= NC) break;
      tmem_wait_chunks<1>(vb);
      if (c + 2 < NC) tmem_ld_chunks<1>(taddr + (c + 2) * 32, va);
      relu_dot<1>(vb, w + (c + 1) * 32, acc);
      if (c + 2 < NC) tmem_wait_chunks<1>(va);
    }
    return sum8(acc);
  } else {
    uint32_t v[1][32];
    tmem_ld_chunks<1>(taddr, v);
    tmem_wait_chunks<1>(v);
    float b[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int jj = 0; jj < HT; jj += 4) {
      const float4 wv = *reinterpret_cast<const float4*>(w + jj);
      b[0] = fmaf(wv.x, fmaxf(__uint_as_float(v[0][jj + 0]), 0.f), b[0]);
      b[1] = fmaf(wv.y, fmaxf(__uint_as_float(v[0][jj + 1]), 0.f), b[1]);
      b[2] = fmaf(wv.z, fmaxf(__uint_as_float(v[0][jj + 2]), 0.f), b[2]);
      b[3] = fmaf(wv.w, fmaxf(__uint_as_float(v[0][jj + 3]), 0.f), b[3]);
    }
    return (b[0] + b[1]) + (b[2] + b[3]);
  }
}

// 320 threads: ten warps over four sub-partitions of 16K registers each allow
// at most 168 registers per thread.
template <MmaKind KIND, bool SPLIT, int HT, int GATHER, bool DOSA = false>
__global__ void __launch_bounds__(kScanThreads, 1)
    scan_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                const ScanArgs a) {
  using Cfg = ScanCfg<KIND>;
  constexpr int PARTS = SPLIT ? 2 : 1;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte aligned base; plain pointer arithmetic on the __shared__ array
  // keeps the shared address space visible to the compiler (LDS/ATOMS, not generic)
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int qcols = a.qcols;                                // Q-tile rows per group
  const int QT = a.QG * a.G;
  uint8_t* Qs = smem;                                       // [G][A][qcols x 128B]
  const int q_bytes = a.G * Cfg::A * qcols * 128;
  const int KS = a.kstages, NS = a.tstages;
  // key tiles per K stage / accumulator unit: 2 only for e4m3 keys (decode), so
  // every other kind compiles with a constant 1
  constexpr bool kPairs = KIND == MmaKind::E4M3 && GATHER == 0;
  const int KT = kPairs && a.kt > 1 ? 2 : 1;
  uint8_t* Ks = smem + ((q_bytes + 1023) & ~1023);          // [KS][KT][A][128 x 128B]
  // streaming rows: per-row histograms [QT][768]; gathered rows: the row's
  // candidate composites [kMaxGatherKeys]
  uint32_t* hist = reinterpret_cast<uint32_t*>(Ks + KS * KT * Cfg::KTILE_BYTES);
  uint64_t* cand = reinterpret_cast<uint64_t*>(hist);                 // [kMaxGatherKeys]
  uint32_t* ghist = reinterpret_cast<uint32_t*>(cand + kMaxGatherKeys);  // [kGatherBins]
  uint64_t* gbnd = reinterpret_cast<uint64_t*>(ghist + kGatherBins);   // [kGatherBoundary]
  ScanSmemTail* T = reinterpret_cast<ScanSmemTail*>(
      GATHER != 0 ? reinterpret_cast<uint8_t*>(gbnd + kGatherBoundary)
                  : reinterpret_cast<uint8_t*>(hist + QT * kHistWords));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool modeB = (a.QG == 1);  // one query per group: halves take alternate stages

  if (threadIdx.x == 0) {
    for (int i = 0; i < KS; ++i) {
      mbar_init(&T->k_full[i], 1);
      mbar_init(&T->k_empty[i], 1);
    }
    mbar_init(&T->q_full, 1);
    mbar_init(&T->q_empty, 1);
    mbar_init(&T->drain, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&T->t_full[s], 1);
      mbar_init(&T->t_empty[s], modeB ? 4 : 8);
    }
    T->abort = 0;
    T->dosa_skips = 0u;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&T->tmem_base, NS * a.stage_cols);
    tmem_relinquish();
  }
  if (warp == kProducerWarp && lane == 0) {
    prefetch_tmap(&qmap);
    prefetch_tmap(&kmap);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = T->tmem_base;
  volatile int* abort = &T->abort;
  const int grid = gridDim.x;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer --
    // Lane 0 owns the barriers; for gathered keys the whole warp reads the
    // row's list (four entries or one block per lane) and issues the copies.
    uint32_t kcount = 0, it = 0;
    bool ok = true;
    for (int round = 0; ok; ++round) {
      const int item = sched_item(round, blockIdx.x, grid);
      if (item >= a.n_items) break;
      ItemGeom g = item_geom<GATHER>(a, item);
      if (g.ntiles == 0) continue;
      if (lane == 0) {
        ok = mbar_wait(&T->q_empty, (it & 1) ^ 1, abort, a.status, 1, a.wait_cycles);
        if (ok) {
          mbar_arrive_expect_tx(&T->q_full, q_bytes);
          // split-query rows: the hi parts of all rows come first, then the lo parts
          const int qrow0 = (g.b * a.q_stride + a.q_off + g.row0) * a.H;
          const int lo_rows = a.batch * a.q_stride * a.H;
          const int part_cols = qcols / PARTS;
          for (int gg = 0; gg < a.G; ++gg)
            for (int at = 0; at < Cfg::A; ++at)
              for (int pt = 0; pt < PARTS; ++pt)
                tma_load_2d(Qs + ((gg * Cfg::A + at) * qcols + pt * part_cols) * 128, &qmap,
                            &T->q_full, at * Cfg::EPA, qrow0 + gg * a.QG * a.H + pt * lo_rows);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      ++it;
      const int krow0 = g.b * a.n_k;
      const int32_t* lst = GATHER != 0
          ? a.klist + ((int64_t)g.b * a.n_q + g.row0) * a.klist_len : nullptr;
      const int nk = (g.ntiles + KT - 1) / KT;                // K stages of this item
      for (int t = 0; t < nk; ++t) {
        const int slot = kcount % KS;
        const uint32_t ph = (kcount / KS) & 1;
        // list entries of this tile (loaded before the wait so their latency overlaps it)
        int rr[4] = {0, 0, 0, 0};
        int ybox = -1;
        // list entries outside [-1, n_k) (never written by this library's own
        // selects) are recorded and read as empty slots
        if constexpr (GATHER == 1) {
          // lane L holds tile rows 2 (L % 16) + L / 16 + 32 j (j = 0..3): the rows
          // that the copies below need from it, one register per copy round
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int e = t * 128 + 2 * (lane & 15) + (lane >> 4) + 32 * j;
            int kk = e < a.klist_len ? lst[e] : -1;
            if (kk < -1 || kk >= a.n_k) {
              set_status(a.status, DSA_ERR_INTERNAL, 111);
              kk = -1;
            }
            rr[j] = krow0 + (kk >= 0 ? kk : 0);
          }
        } else if constexpr (GATHER == 2) {
          const int bs = 1 << a.lb_shift;
          const int box = bs < 128 ? bs : 128;
          if (lane < 128 / box) {
            const int e = t * 128 + lane * box;            // token slot in the row's list
            const int slot_b = e >> a.lb_shift;
            int blk = slot_b < a.klist_len ? lst[slot_b] : -1;
            if (blk < -1 || (long long)blk * bs >= a.n_k) {
              set_status(a.status, DSA_ERR_INTERNAL, 112);
              blk = -1;
            }
            // an empty slot loads a box wholly before row 0: zero fill, no traffic
            ybox = blk >= 0 ? krow0 + blk * bs + (e & (bs - 1)) : -box;
          }
        }
        // tiles of this stage inside the item (a ragged last stage loads one)
        const int nvalid = kPairs ? min(KT, g.ntiles - t * KT) : 1;
        // DSA_FLAG_TEST_STALL: this stage is counted but never loaded, so the MMA
        // warp's bounded wait on it runs out and the abort path runs
        const bool stall = GATHER == 0 && a.test_stall && blockIdx.x == 0 && it == 1 && t == 1;
        if (lane == 0) {
          ok = mbar_wait(&T->k_empty[slot], ph ^ 1, abort, a.status, 2, a.wait_cycles);
          if (ok && !stall && GATHER != 1)
            mbar_arrive_expect_tx(&T->k_full[slot], nvalid * Cfg::KTILE_BYTES);
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        if (stall) {
          ++kcount;
          continue;
        }
        if constexpr (GATHER == 0) {
          if (lane == 0) {
            for (int j = 0; j < nvalid; ++j) {
              const int tstart = (g.t_hi - (t * KT + j)) << 7;
              for (int at = 0; at < Cfg::A; ++at)
                tma_load_2d(Ks + ((slot * KT + j) * Cfg::A + at) * 16384, &kmap, &T->k_full[slot],
                            at * Cfg::EPA, krow0 + tstart);
            }
          }
        } else if constexpr (GATHER == 1) {
          // arbitrary key rows: 16-byte asynchronous copies, two whole 256-byte
          // rows per warp instruction (lane = row parity x 16-byte chunk), into
          // the 128-byte swizzled layout the MMA reads.  In round i lanes 0-15
          // copy tile row 2i and lanes 16-31 row 2i + 1, whose entries lanes
          // i % 16 and 16 + i % 16 hold in register i / 16.  The stage's barrier
          // completes once every lane's copies have landed and lane 0 arrived.
          static_assert(Cfg::A == 2, "bf16 key rows");
          const int ch = lane & 15, at = ch >> 3, cc = ch & 7, odd = lane >> 4;
          uint8_t* kb = Ks + (slot * Cfg::A + at) * 16384;
          const uint8_t* kg = reinterpret_cast<const uint8_t*>(a.kraw) + ch * 16;
#pragma unroll
          for (int i = 0; i < 64; ++i) {
            const int v = __shfl_sync(0xffffffffu, rr[i >> 4], (i & 15) + 16 * odd);
            const int r = 2 * i + odd;
            cp_async_16(kb + r * 128 + ((cc ^ (r & 7)) << 4), kg + (size_t)v * 256);
          }
          cp_async_mbar_arrive(&T->k_full[slot]);
          __syncwarp();
          if (lane == 0) mbar_arrive(&T->k_full[slot]);
        } else {
          // runs of 2^lb_shift consecutive keys (box of min(bs, 128) rows)
          const int bs = 1 << a.lb_shift;
          const int box = bs < 128 ? bs : 128;
          if (lane < 128 / box)
            for (int at = 0; at < Cfg::A; ++at)
              tma_load_2d(Ks + (slot * Cfg::A + at) * 16384 + lane * box * 128, &kmap,
                          &T->k_full[slot], at * Cfg::EPA, ybox);
        }
        ++kcount;
      }
    }
    if (lane == 0 && *abort) {
      // abort path: let this CTA's own copies in flight land before exit
      if (it > 0) mbar_wait_drain(&T->q_full, (it - 1) & 1, a.wait_cycles);
      for (uint32_t i = kcount > (uint32_t)KS ? kcount - KS : 0; i < kcount; ++i)
        mbar_wait_drain(&T->k_full[i % KS], (i / KS) & 1, a.wait_cycles);
    }
  } else if (warp == kMmaWarp) {
    // ----------------------------------------------------------------- MMA --
    if (lane == 0) {
      // split-query rows: the hi and lo parts are two MMAs into one accumulator
      const int ncols = qcols / PARTS;
      const uint32_t idesc = make_idesc<KIND>(ncols);
      uint32_t kcount = 0, ucount = 0, it = 0;
      bool ok = true;
      for (int round = 0; ok; ++round) {
        const int item = sched_item(round, blockIdx.x, grid);
        if (item >= a.n_items) break;
        ItemGeom g = item_geom<GATHER>(a, item);
        if (g.ntiles == 0) continue;
        if (!mbar_wait(&T->q_full, it & 1, abort, a.status, 3, a.wait_cycles)) break;
        ++it;
        tc_fence_after();
        const int nunits = (g.ntiles + KT - 1) / KT * a.G;
        for (int u = 0; u < nunits; ++u) {
          const int gg = u & (a.G - 1);
          const int slot = kcount % KS;
          if (gg == 0) {
            if (!mbar_wait(&T->k_full[slot], (kcount / KS) & 1, abort, a.status, 4, a.wait_cycles)) { ok = false; break; }
            // rows written by 16-byte asynchronous copies (generic proxy): order
            // them before the tensor core's reads
            if constexpr (GATHER == 1) fence_proxy_async_smem();
          }
          const int s = ucount % NS;
          if (!mbar_wait(&T->t_empty[s], ((ucount / NS) & 1) ^ 1, abort, a.status, 5, a.wait_cycles)) { ok = false; break; }
          tc_fence_after();
          const uint32_t qbase = smem_u32(Qs + gg * Cfg::A * qcols * 128);
          // one accumulator block of ncols columns per key tile of the stage
          const int nvalid = kPairs ? min(KT, g.ntiles - (u / a.G) * KT) : 1;
          for (int j = 0; j < nvalid; ++j) {
            const uint32_t d = tmem_base + s * a.stage_cols + j * ncols;
            const uint32_t kbase = smem_u32(Ks + (slot * KT + j) * Cfg::A * 16384);
#pragma unroll
            for (int at = 0; at < Cfg::A; ++at) {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint64_t ad = make_sdesc(kbase + at * 16384 + kk * 32);
#pragma unroll
                for (int pt = 0; pt < PARTS; ++pt) {
                  const uint64_t bd = make_sdesc(qbase + (at * qcols + pt * ncols) * 128 + kk * 32);
                  tc_mma<KIND>(d, ad, bd, idesc, (at | kk | pt) != 0);
                }
              }
            }
          }
          tc_commit(&T->t_full[s]);
          if (gg == a.G - 1) {
            tc_commit(&T->k_empty[slot]);
            ++kcount;
          }
          ++ucount;
        }
        if (!ok) break;
        tc_commit(&T->q_empty);
      }
      if (!ok) {
        // abort path: wait for the MMAs already issued before TMEM is freed
        tc_commit(&T->drain);
        mbar_wait_drain(&T->drain, 0, a.wait_cycles);
      }
    }
  } else if constexpr (GATHER != 0) {
    // ------------------------------------------ epilogue, gathered keys --
    // One query row per item; the halves take alternate accumulator stages.
    // Every candidate's composite goes to shared memory (list position e);
    // at the end of the row one exact selection keeps its top `keep`, written
    // to the row's first sub-log.
    const int etid = threadIdx.x;
    const int quad = warp & 3;
    const int half = warp >> 2;
    uint32_t ucount = 0;
    int step_par = 0;
    for (int round = 0;; ++round) {
      const int item = sched_item(round, blockIdx.x, grid);
      if (item >= a.n_items) break;
      ItemGeom g = item_geom<GATHER>(a, item);
      const int pos0 = (a.q_pos0 ? a.q_pos0[g.b] : a.n_tok - a.q_stride) + a.q_off;
      const int klen = a.k_len ? a.k_len[g.b] : a.n_tok;
      const int64_t slot0 = (int64_t)g.b * a.n_q + g.row0;     // one key chunk
      const int nkeys = g.kend;                                 // list length in tokens
      const int nleg = g.nrows > 0 ? max(0, min(pos0 + g.row0, klen - 1) + 1) : 0;
      const int32_t* lst = a.klist + slot0 * a.klist_len;
      const int64_t grow = (int64_t)g.b * a.q_stride + a.q_off + g.row0;
      for (int i = etid; i < HT; i += kEpiThreads) T->wsm[i] = g.nrows > 0 ? a.w[grow * HT + i] : 0.f;
      for (int i = etid; i < kGatherBins; i += kEpiThreads) ghist[i] = 0u;
      if (etid == 0) {
        T->gather_legal = 0;
        T->gather_nwin = 0;
        T->gather_nbnd = 0;
      }
      named_bar_sync(kBarEpi, kEpiThreads);
      int legal_cnt = 0;
      float lo = __int_as_float(0x7f800000), hi = -__int_as_float(0x7f800000);
      // this lane's key at list position e of unit u (a global load)
      auto key_at = [&](int u) -> int {
        const int e = u * 128 + quad * 32 + lane;
        if constexpr (GATHER == 1) {
          return e < a.klist_len ? lst[e] : -1;
        } else {
          const int sb = e >> a.lb_shift;
          const int blk = sb < a.klist_len ? lst[sb] : -1;
          return blk >= 0 ? (blk << a.lb_shift) + (e & ((1 << a.lb_shift) - 1)) : -1;
        }
      };
      // this half takes every other unit; the key of its next unit is loaded one
      // unit ahead so the list lookup never waits on memory
      const int u0 = (int)((ucount + half) & 1);
      int key_next = u0 < g.ntiles ? key_at(u0) : -1;
      for (int u = u0; u < g.ntiles; u += 2) {
        const uint32_t uc = ucount + u;
        const int s = uc % NS;
        const int e = u * 128 + quad * 32 + lane;
        const int key = key_next;
        if (u + 2 < g.ntiles) key_next = key_at(u + 2);
        const bool got = mbar_wait(&T->t_full[s], (uc / NS) & 1, abort, a.status, 6, a.wait_cycles);
        __syncwarp();
        if (!__all_sync(0xffffffffu, got)) continue;
        tc_fence_after();
        const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16) + s * a.stage_cols;
        const float acc = row_acc<HT>(taddr, T->wsm);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&T->t_empty[s]);
        const bool legal = (unsigned)key < (unsigned)nleg;
        legal_cnt += legal ? 1 : 0;
        if (legal) {
          lo = fminf(lo, acc);
          hi = fmaxf(hi, acc);
        }
        if (e < nkeys) cand[e] = legal ? make_comp(acc, key) : 0ull;
      }
      ucount += g.ntiles;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        legal_cnt += __shfl_xor_sync(0xffffffffu, legal_cnt, off);
        lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, off));
        hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, off));
      }
      if (lane == 0) {
        if (legal_cnt) atomicAdd(&T->gather_legal, legal_cnt);
        T->gather_lo[warp] = lo;
        T->gather_hi[warp] = hi;
      }
      if (etid == 0) T->epi_stop[step_par] = *abort;   // uniform stop decision
      named_bar_sync(kBarEpi, kEpiThreads);
      const bool stop = T->epi_stop[step_par] != 0;
      step_par ^= 1;
      if (stop) break;
      const int n_legal = T->gather_legal;
      const int ncand = nkeys < kMaxGatherKeys ? nkeys : kMaxGatherKeys;
      uint64_t* out = a.logs + slot0 * a.nsub * a.capw;
      int cnt = 0;
      bool radix = false;
      if (n_legal > a.keep) {
        // Linear score bins over [lo, hi]: count, locate the bin holding the keep-th
        // best, emit every candidate above it and rank that bin's candidates exactly.
        // A crowded bin is split once more into its own linear bins; only a bin that
        // stays crowded (long runs of equal scores) falls back to the radix select.
        float lo2 = T->gather_lo[0], hi2 = T->gather_hi[0];
#pragma unroll
        for (int w = 1; w < kEpiWarps; ++w) {
          lo2 = fminf(lo2, T->gather_lo[w]);
          hi2 = fmaxf(hi2, T->gather_hi[w]);
        }
        const float span = hi2 - lo2;
        const float scale0 = span > 0.f ? (float)(kGatherBins - 1) / span : 0.f;
        auto bin_at = [&](uint64_t c, float base, float sc) {
          const int b = __float2int_rz((key_score((uint32_t)(c >> 32)) - base) * sc);
          return min(kGatherBins - 1, max(0, b));
        };
        int need = a.keep;          // still to emit
        int emitted = 0;            // winners already in out[]
        int scope_bin = -1;         // level 1: only candidates of this level-0 bin
        float base = lo2, scale = scale0;
        bool done = false;
        for (int level = 0; level < 2 && !done && !radix; ++level) {
          if (level == 1) {
            for (int i = etid; i < kGatherBins; i += kEpiThreads) ghist[i] = 0u;
            if (etid == 0) {
              T->gather_nwin = 0;
              T->gather_nbnd = 0;
            }
            named_bar_sync(kBarEpi, kEpiThreads);
          }
          auto in_scope = [&](uint64_t c) {
            return c != 0ull && (scope_bin < 0 || bin_at(c, lo2, scale0) == scope_bin);
          };
          for (int e = etid; e < ncand; e += kEpiThreads) {
            const uint64_t c = cand[e];
            if (in_scope(c)) atomicAdd(&ghist[bin_at(c, base, scale)], 1u);
          }
          named_bar_sync(kBarEpi, kEpiThreads);
          // thread t owns the 16 bins from 4095 - 16 t downwards; scan in that order
          uint32_t own = 0;
#pragma unroll
          for (int i = 0; i < 16; ++i) own += ghist[kGatherBins - 1 - 16 * etid - i];
          uint32_t incl = own;
#pragma unroll
          for (int off = 1; off < 32; off <<= 1) {
            const uint32_t o = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += o;
          }
          uint32_t* wsum = reinterpret_cast<uint32_t*>(T->sel.hist);
          if (lane == 31) wsum[warp] = incl;
          named_bar_sync(kBarEpi, kEpiThreads);
          uint32_t wbase = 0;
          for (int w = 0; w < warp; ++w) wbase += wsum[w];
          const uint32_t excl = wbase + incl - own;
          if (excl < (uint32_t)need && (uint32_t)need <= excl + own) {
            uint32_t cum = excl;
            for (int i = 0; i < 16; ++i) {
              const int b = kGatherBins - 1 - 16 * etid - i;
              const uint32_t c = ghist[b];
              if (cum + c >= (uint32_t)need) {
                T->sel.sel[2] = b;
                T->sel.sel[3] = (int)cum;          // in-scope candidates strictly above bin b
                break;
              }
              cum += c;
            }
          }
          named_bar_sync(kBarEpi, kEpiThreads);
          const int bstar = T->sel.sel[2], above = T->sel.sel[3];
          for (int e0 = 0; e0 < ncand; e0 += kEpiThreads) {
            const int e = e0 + etid;
            const uint64_t c = e < ncand ? cand[e] : 0ull;
            const int b = in_scope(c) ? bin_at(c, base, scale) : -1;
            const bool win = b > bstar, edge = b == bstar;
            const unsigned bw = __ballot_sync(0xffffffffu, win);
            const unsigned be = __ballot_sync(0xffffffffu, edge);
            int pw = 0, pe = 0;
            if (lane == 0) {
              if (bw) pw = atomicAdd(&T->gather_nwin, __popc(bw));
              if (be) pe = atomicAdd(&T->gather_nbnd, __popc(be));
            }
            pw = __shfl_sync(0xffffffffu, pw, 0);
            pe = __shfl_sync(0xffffffffu, pe, 0);
            const unsigned lt = (1u << lane) - 1u;
            if (win) out[emitted + pw + __popc(bw & lt)] = c;
            if (edge) {
              const int sl = pe + __popc(be & lt);
              if (sl < kGatherBoundary) gbnd[sl] = c;
            }
          }
          named_bar_sync(kBarEpi, kEpiThreads);
          const int nb = T->gather_nbnd;
          emitted += above;
          need -= above;
          if (nb <= kGatherBoundary) {
            if (warp == 0) warp_take_top(gbnd, nb, need, out, emitted, lane);
            cnt = a.keep;
            done = true;
          } else if (level == 0 && scale0 > 0.f) {
            // split the crowded bin: its scores lie in [lo + b / scale, lo + (b + 1) / scale)
            scope_bin = bstar;
            base = lo2 + (float)bstar / scale0;
            scale = scale0 * (float)(kGatherBins - 1);
          } else {
            radix = true;                                // equal scores: exact radix
          }
        }
      }
      if (n_legal > 0 && (n_legal <= a.keep || radix)) {
        const uint64_t* segs[1] = {cand};
        const int segn[1] = {ncand};
        uint64_t thr = 1ull;                          // every legal composite is >= 1
        if (n_legal > a.keep)
          thr = radix_select<kEpiThreads>(segs, segn, 1, a.keep, &T->sel, etid, kBarEpi);
        cnt = compact_ge<kEpiThreads>(segs, segn, 1, thr, out, &T->sel, etid, kBarEpi, nullptr);
      }
      if (etid < a.nsub) a.log_cnt[slot0 * a.nsub + etid] = etid == 0 ? cnt : 0;
      if (etid == 0) a.log_thr[slot0] = 0ull;
      named_bar_sync(kBarEpi, kEpiThreads);             // cand is reused by the next row
    }
  } else {
    // ------------------------------------------------------------ epilogue --
    const int etid = threadIdx.x;              // 0..255
    const int quad = warp & 3;                 // TMEM lane quadrant
    const int half = warp >> 2;                // column half / stage (mode B)
    const int sub = modeB ? warp : quad;       // this warp's sub-log index
    constexpr int H = HT;
    const int hshift = 31 - __clz(H);          // log2(H)
    const int qhalf = modeB ? 1 : (a.QG >> 1); // query rows per warp per group
    uint32_t ucount = 0;
    int step_par = 0;
    bool stop = false;
    uint32_t dosa_n = 0;                       // DoSA: (row, unit) pairs this warp skipped
    // DoSA: check the block bounds only where they are seen to bite (the seeds
    // alone rule out at least 1/32 of the blocks); otherwise the per-unit checks
    // would cost more than they save (the seeded thresholds still apply)
    bool dosa_on = false;
    if constexpr (DOSA) dosa_on = a.dosa_counts[1] * 32ull >= a.dosa_counts[0] && a.dosa_counts[1] > 0;
    for (int round = 0; !stop; ++round) {
      const int item = sched_item(round, blockIdx.x, grid);
      if (item >= a.n_items) break;
      ItemGeom g = item_geom<GATHER>(a, item);
      // DoSA: per query group, the bound block of the cached skip decision
      // (decided once per block, on entering it, with the thresholds of then)
      int dblk0 = -1, dblk1 = -1;
      unsigned dmask0 = 0u, dmask1 = 0u;
      const int pos0 = (a.q_pos0 ? a.q_pos0[g.b] : a.n_tok - a.q_stride) + a.q_off;
      const int klen = a.k_len ? a.k_len[g.b] : a.n_tok;
      const int64_t slot0 = ((int64_t)g.b * a.n_q + g.row0) * a.C + g.c;  // slot of row 0
      // ---- item init: row states, histograms, head weights
      for (int r = etid; r < QT; r += kEpiThreads) {
        unsigned long long thr0 = 0ull;
        if constexpr (DOSA) {
          // the seed set's guarantee: keep legal keys score at least the seed, so
          // a threshold at its key (index part 0) drops none of the keep best
          if (r < g.nrows) {
            const float sd = a.dosa_seed[(int64_t)g.b * a.q_stride + a.q_off + g.row0 + r];
            if (sd != -__int_as_float(0x7f800000)) thr0 = (unsigned long long)score_key(sd) << 32;
          }
        }
        T->row_thr[r] = thr0;
        T->row_b1[r] = -1;
        T->row_raise[r] = 0;
        int nleg = 0;
        if (r < g.nrows) {
          const int pos = pos0 + g.row0 + r;
          if (a.bs_shift > 0)
            nleg = max(0, min(min(pos + 1, klen) >> a.bs_shift, g.kend) - g.kbeg);
          else
            nleg = max(0, min(min(pos, klen - 1), g.kend - 1) - g.kbeg + 1);
        }
        T->row_nleg[r] = nleg;
        // positions grow with the row, so row 0 has the item's smallest legal
        // count; an item with unused row slots (nleg 0) has none that is always legal
        if (r == 0) T->item_min_nleg = g.nrows < QT ? 0 : nleg;
#pragma unroll
        for (int w8 = 0; w8 < 8; ++w8) T->subcnt[r][w8] = 0;
      }
      for (int i = etid; i < QT * kHistWords; i += kEpiThreads) hist[i] = 0u;
      for (int i = etid; i < QT * H; i += kEpiThreads) {
        const int r = i >> hshift, j = i & (H - 1);
        float wv = 0.f;
        if (r < g.nrows) {
          const int64_t grow = (int64_t)g.b * a.q_stride + a.q_off + g.row0 + r;
          wv = a.w[grow * H + j];
          if (a.row_scale) wv *= a.row_scale[grow];
          if (a.head_scale) wv *= a.head_scale[grow * H + j];
        }
        T->wsm[i] = wv;
      }
      if (etid == 0) T->raise_any = 0;
      named_bar_sync(kBarEpi, kEpiThreads);
      const int nunits = (g.ntiles + KT - 1) / KT * a.G;
      auto ks_at = [&](int uu) -> float {
        if (!a.k_scale) return 1.f;
        const int key = ((g.t_hi - (uu >> (a.G - 1)) * KT) << 7) + quad * 32 + lane;
        return key < a.n_k ? a.k_scale[(int64_t)g.b * a.n_k + key] : 1.f;
      };
      // scale of the second key tile of a unit (below the first; may precede the
      // item's first tile in a ragged last unit)
      auto ks_at1 = [&](int uu) -> float {
        if (!a.k_scale) return 1.f;
        const int key = ((g.t_hi - (uu >> (a.G - 1)) * KT - 1) << 7) + quad * 32 + lane;
        return key >= 0 && key < a.n_k ? a.k_scale[(int64_t)g.b * a.n_k + key] : 1.f;
      };
      const int ustep = modeB ? 2 : 1;                  // this warp's units: every / every other
      const int ufirst = modeB ? (int)((ucount + half) & 1) : 0;
      float ks_next = ufirst < nunits ? ks_at(ufirst) : 1.f;
      float ks_next1 = 1.f;
      if constexpr (kPairs) ks_next1 = ufirst < nunits && KT > 1 ? ks_at1(ufirst) : 1.f;
      int u = 0;
      int steps = 0;
      while (u < nunits) {
        // one step = up to two units (stage 0 / stage 1)
        const int nstep = min(2, nunits - u);
        for (int v = 0; v < nstep; ++v) {
          const int uu = u + v;
          const uint32_t uc = ucount + v;
          const int s = uc % NS;
          const bool mine = modeB ? (half == (int)(uc & 1)) : true;
          if (!mine) continue;
          const int gg = uu & (a.G - 1);
          const int t = uu >> (a.G - 1);
          const int key = ((g.t_hi - t * KT) << 7) + quad * 32 + lane;
          // key dequant scale: loaded one unit of this warp ahead
          const float ks = ks_next;
          if (uu + ustep < nunits) ks_next = ks_at(uu + ustep);
          float ks1 = 1.f;
          if constexpr (kPairs) {
            ks1 = ks_next1;
            if (KT > 1 && uu + ustep < nunits) ks_next1 = ks_at1(uu + ustep);
          }
          // DoSA bounds of this warp's rows over the tile's bound block (rows past
          // the item and rows of an unbounded problem: +inf, never skipped)
          // DoSA: on entering a bound block, this warp's rows' bounds over it
          // (loaded before the wait; rows past the item: +inf, never skipped)
          float ubv[4];
          unsigned skipm = 0u;
          bool dfresh = false;
          int dblk = 0;
          if constexpr (DOSA) if (dosa_on) {   // heads >= 32: at most four rows per warp
            dblk = ((g.t_hi - t * KT) << 7) >> a.dosa_shift;
            dfresh = dblk != (gg ? dblk1 : dblk0);
            if (dfresh) {
              const int rb = gg * a.QG + (modeB ? 0 : half * qhalf);
              const int64_t gr = (int64_t)g.b * a.q_stride + a.q_off + g.row0 + rb;
#pragma unroll
              for (int qi = 0; qi < 4; ++qi)
                ubv[qi] = qi < qhalf && rb + qi < g.nrows
                              ? __ldg(a.dosa_ub + (gr + qi) * a.dosa_nblk + dblk)
                              : __int_as_float(0x7f800000);
            }
          }
          const bool got = mbar_wait(&T->t_full[s], (uc / NS) & 1, abort, a.status, 6, a.wait_cycles);
          __syncwarp();
          if (!__all_sync(0xffffffffu, got)) continue;
          tc_fence_after();
          const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16) + s * a.stage_cols;
          // queries handled by this warp inside group gg
          const int qbeg = modeB ? 0 : half * qhalf;
          const int rbase = gg * a.QG + qbeg;          // first item row of this warp
          FilterCtx fc;
          fc.key = key;
          fc.ks = ks;
          fc.kbeg = g.kbeg;
          fc.lane = lane;
          fc.lanemask_lt = (1u << lane) - 1u;
          fc.sub = sub;
          fc.logs = a.logs + (slot0 * a.nsub + sub) * a.capw;
          fc.row_stride = (uint32_t)(a.C * a.nsub * a.capw);
          fc.all_legal = key - (int)(quad * 32 + lane) >= g.kbeg &&
                         key - (int)(quad * 32 + lane) + 127 - g.kbeg < T->item_min_nleg;
          fc.hist = hist;
          fc.T = T;
          fc.capw = a.capw;
          fc.status = a.status;
          if constexpr (DOSA) if (dosa_on) {
            // DoSA: a row whose upper bound over the tile's block lies below its
            // threshold (a lower bound of its final keep-th best) has no candidate
            // the filter could keep in the block; its head sums are skipped.  A
            // threshold raised inside the block only prunes from the next one.
            if (dfresh) {
              unsigned m = 0u;
#pragma unroll
              for (int qi = 0; qi < 4; ++qi) {
                if (qi >= qhalf) break;
                const unsigned long long th = T->row_thr[rbase + qi];
                if (th != 0ull && ubv[qi] < key_score((uint32_t)(th >> 32))) m |= 1u << qi;
              }
              if (gg) { dblk1 = dblk; dmask1 = m; } else { dblk0 = dblk; dmask0 = m; }
            }
            skipm = gg ? dmask1 : dmask0;
            if (skipm != 0u) {
              dosa_n += __popc(skipm);
              for (int qi = 0; qi < qhalf; ++qi)
                if (!((skipm >> qi) & 1u))
                  unit_heads_n<HT, 1>(fc, taddr + (qbeg + qi) * HT, &T->wsm[(rbase + qi) * HT],
                                      rbase + qi);
            }
          }
          if (DOSA && skipm != 0u) {
            // (pruned rows handled above)
          } else if constexpr (HT >= 32) {
            if (qhalf == 2)
              unit_heads_n<HT, 2>(fc, taddr + qbeg * HT, &T->wsm[rbase * HT], rbase);
            else if (qhalf == 1)
              unit_heads_n<HT, 1>(fc, taddr + qbeg * HT, &T->wsm[rbase * HT], rbase);
            else
              unit_heads<HT>(fc, taddr + qbeg * HT, &T->wsm[rbase * HT], qhalf, rbase);
          } else {
            if (qhalf == 8)
              unit_heads_small<HT, 8>(fc, taddr + qbeg * HT, &T->wsm[rbase * HT], rbase);
            else
              unit_heads<HT>(fc, taddr + qbeg * HT, &T->wsm[rbase * HT], qhalf, rbase);
          }
          if constexpr (kPairs) {
            // the unit's second key tile (one query row per item: mode B, qhalf 1),
            // in the next ncols accumulator columns; absent in a ragged last unit
            if (KT > 1 && t * KT + 1 < g.ntiles) {
              const int key1 = key - 128;
              fc.key = key1;
              fc.ks = ks1;
              fc.all_legal = key1 - (int)(quad * 32 + lane) >= g.kbeg &&
                             key1 - (int)(quad * 32 + lane) + 127 - g.kbeg < T->item_min_nleg;
              const uint32_t tcol = taddr + qcols / PARTS;
              if constexpr (HT >= 32)
                unit_heads_n<HT, 1>(fc, tcol, &T->wsm[rbase * HT], rbase);
              else
                unit_heads<HT>(fc, tcol, &T->wsm[rbase * HT], 1, rbase);
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&T->t_empty[s]);
        }
        ucount += nstep;
        u += nstep;
        ++steps;
        // ---- compaction of this warp's own sub-logs that near capacity (no barrier:
        // only this warp writes them; thr may be raised concurrently, which only
        // keeps fewer entries, all still >= a valid threshold)
        for (int gg = 0; gg < a.G; ++gg) {
          for (int qi = 0; qi < qhalf; ++qi) {
            const int r = gg * a.QG + (modeB ? 0 : half * qhalf) + qi;
            if (r >= g.nrows) continue;
            const int n = T->subcnt[r][sub];
            if (n <= a.capw - kCompactSlack) continue;
            uint64_t* lg = a.logs + ((slot0 + (int64_t)r * a.C) * a.nsub + sub) * a.capw;
            const int kept = compact_sublog(lg, n, T->row_thr[r], lane);
            if (lane == 0) {
              T->subcnt[r][sub] = kept;
              if (kept > a.capw - kCompactSlack) T->raise_any = T->row_raise[r] = 1;
            }
            __syncwarp();
          }
        }
        // ---- every kUpdateSteps steps (and at the item end): threshold update
        const bool last = u >= nunits;
        if (!last && (steps & (kUpdateSteps - 1)) != 0) continue;
        // uniform decisions: thread 0 snapshots the abort and raise flags before the
        // barrier (a raise flagged after the snapshot waits for the next update)
        if (etid == 0) {
          T->epi_stop[step_par] = *abort;
          T->raise_snap[step_par] = T->raise_any;
        }
        named_bar_sync(kBarEpi, kEpiThreads);
        stop = T->epi_stop[step_par] != 0;
        const bool do_raise = T->raise_snap[step_par] != 0;
        step_par ^= 1;
        if (stop) break;
        // one warp per row, from the row's histograms
        for (int r = warp; r < g.nrows; r += kEpiWarps) {
          uint32_t* h = hist + r * kHistWords;
          int above1;
          const int nb1 = hist_find(h, 0, a.keep, lane, &above1);
          if (nb1 < 0) continue;                           // fewer than keep kept so far
          const int ob1 = T->row_b1[r];
          if (nb1 != ob1) {
            if (ob1 >= 0 && nb1 == ob1 + 1) {
              // the upper fine histogram becomes the lower one
              for (int i = lane; i < 256; i += 32) {
                h[256 + i] = h[512 + i];
                h[512 + i] = 0u;
              }
            } else {
              // first threshold or a jump: the fine histograms restart empty and count
              // the candidates kept from now on (low counts: a looser, valid threshold)
              for (int i = lane; i < 512; i += 32) h[256 + i] = 0u;
            }
            __syncwarp();
            if (lane == 0) T->row_b1[r] = nb1;
          }
          __syncwarp();
          int above2;
          const int b2 = hist_find(h + 256, above1, a.keep, lane, &above2);
          if (lane == 0) {
            // the keep-th best lies in top-byte bin nb1, and in its fine bin b2 when the
            // fine counts reach it
            const uint32_t hi = b2 >= 0 ? (((uint32_t)nb1 << 24) | ((uint32_t)b2 << 16))
                                        : ((uint32_t)nb1 << 24);
            const unsigned long long thr = (unsigned long long)hi << 32;
            if (thr > T->row_thr[r]) T->row_thr[r] = thr;
          }
          __syncwarp();
        }
        named_bar_sync(kBarEpi, kEpiThreads);
        if (!do_raise) continue;
        // ---- exact raise (rare: long runs of tied scores)
        for (int r = 0; r < g.nrows; ++r) {
          if (!T->row_raise[r]) continue;
          const int64_t rs = slot0 + (int64_t)r * a.C;
          const uint64_t* segs[8];
          int segn[8];
          int total = 0;
          for (int sb = 0; sb < a.nsub; ++sb) {
            segs[sb] = a.logs + (rs * a.nsub + sb) * a.capw;
            segn[sb] = T->subcnt[r][sb];
            total += segn[sb];
          }
          if (total > a.keep) {
            const uint64_t pfx = radix_select<kEpiThreads>(segs, segn, a.nsub, a.keep, &T->sel, etid, kBarEpi);
            if (etid == 0 && pfx > T->row_thr[r]) T->row_thr[r] = pfx;
          }
          named_bar_sync(kBarEpi, kEpiThreads);
          // the owners of row r's sub-logs compact them with the new threshold
          const bool owner = modeB || ((r % a.QG) / qhalf == half);
          if (owner && T->subcnt[r][sub] > 0) {
            uint64_t* lg = a.logs + (rs * a.nsub + sub) * a.capw;
            const int kept = compact_sublog(lg, T->subcnt[r][sub], T->row_thr[r], lane);
            if (lane == 0) T->subcnt[r][sub] = kept;
            __syncwarp();
          }
          named_bar_sync(kBarEpi, kEpiThreads);
          if (etid == 0) T->row_raise[r] = 0;
          named_bar_sync(kBarEpi, kEpiThreads);
        }
        if (etid == 0) T->raise_any = 0;
        named_bar_sync(kBarEpi, kEpiThreads);
      }
      // ---- item end (split-K): every warp trims its own sub-logs to the final
      // threshold (the last step always ran a threshold update), so the select
      // stage reads about k candidates per key chunk instead of every survivor
      named_bar_sync(kBarEpi, kEpiThreads);
      if (!stop && a.C > 1) {
        for (int gg = 0; gg < a.G; ++gg) {
          for (int qi = 0; qi < qhalf; ++qi) {
            const int r = gg * a.QG + (modeB ? 0 : half * qhalf) + qi;
            if (r >= g.nrows) continue;
            const int n = T->subcnt[r][sub];
            if (n == 0) continue;
            uint64_t* lg = a.logs + ((slot0 + (int64_t)r * a.C) * a.nsub + sub) * a.capw;
            const int kept = compact_sublog(lg, n, T->row_thr[r], lane);
            if (lane == 0) T->subcnt[r][sub] = kept;
            __syncwarp();
          }
        }
      }
      named_bar_sync(kBarEpi, kEpiThreads);
      // ---- item end: publish sub-log fills and thresholds
      for (int r = etid; r < g.nrows; r += kEpiThreads) {
        const int64_t rs = slot0 + (int64_t)r * a.C;
        for (int sb = 0; sb < a.nsub; ++sb) a.log_cnt[rs * a.nsub + sb] = T->subcnt[r][sb];
        a.log_thr[rs] = T->row_thr[r];
      }
      if (etid == 0) T->epi_stop[step_par] = *abort;
      named_bar_sync(kBarEpi, kEpiThreads);
      stop = stop || T->epi_stop[step_par] != 0;
      step_par ^= 1;
    }
    if constexpr (DOSA) {
      // each (row, unit) is counted by the quadrant-0 warp of its half
      if (lane == 0 && quad == 0 && dosa_n) atomicAdd(&T->dosa_skips, dosa_n);
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (DOSA) {
    if (threadIdx.x == 0 && a.dosa_pruned && T->dosa_skips)
      atomicAdd(a.dosa_pruned, (unsigned long long)T->dosa_skips);
  }
  if (warp == kMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, NS * a.stage_cols);
  }
}

}  // namespace dsa

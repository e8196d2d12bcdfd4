// scan.cuh — the indexer scan: tcgen05 scoring tile + fused ReLU / head-weight
// reduction / causal mask + streaming exact top-k filter.
//
// Computes, for every query row t of a work item and every legal key s,
//     I_{t,s} = sum_j w_{t,j} * ReLU(q_{t,j} . k_s)          (DSA indexer score)
// ("PaperTrace 2.2.2 MISA, LISA and ResMiSA", opening DSA definition; the
// kernel fuses score, causal mask and top-k so the n^2 score matrix never
// reaches memory, section 2.2 "kernel boundary").  Restricted to a routed
// head subset this is MISA's step 4 ("MISA: Mixture of Indexer Sparse
// Attention", method step 4): the caller passes gathered q / w rows.
//
// Layout of one CTA (persistent, one work item at a time):
//   warps 0-7  epilogue: TMEM -> registers, ReLU, * w, sum over heads, causal
//              mask, composite key, threshold filter, append to the row's
//              candidate log; exact threshold raises when a log fills
//   warp 8     TMA producer: Q tile of the item (resident), K tiles streamed
//   warp 9     MMA issuer (one thread) + TMEM allocator
// MMA: M = 128 keys (TMEM lane = key), N = query rows x heads (x 2 for the
// split-query fp8 form), K = d; fp32 accumulate in TMEM, two accumulator
// stages so the epilogue of one unit overlaps the MMA of the next.
#pragma once
#include "common.cuh"
#include "select.cuh"

namespace dsa {

struct ScanArgs {
  int32_t batch, n_q, n_k, H, d;
  int32_t keep;          // entries each row must keep (top-k or k')
  int32_t QG;            // query rows per accumulator group (<= 256 / (H * parts))
  int32_t G;             // groups per work item (1 or 2)
  int32_t stage_cols;    // TMEM columns per accumulator stage (128 or 256)
  int32_t n_qt;          // query tiles per sequence (ceil(n_q / (QG*G)))
  int32_t C;             // key chunks per row (split-K); 1 = whole prefix
  int32_t chunk;         // keys per chunk (multiple of 128) when C > 1
  int32_t n_items;       // batch * n_qt * C
  const int32_t* q_pos0; // [batch] or null: n_k - n_q
  const int32_t* k_len;  // [batch] or null: n_k
  const float* w;        // [rows, H]
  const float* row_scale;   // [rows] or null: multiplies w (query dequant scale)
  const float* head_scale;  // [rows, H] or null: multiplies w (split-query part scale)
  const float* k_scale;     // [batch * n_k] or null: multiplies the score (key dequant scale)
  uint64_t* logs;        // [rows * C][2][cap] composite keys
  int32_t* log_cnt;      // [rows * C]
  int32_t* log_buf;      // [rows * C]
  int32_t cap;           // entries per log buffer (>= keep + 256)
  int32_t* status;       // workspace status word
};

constexpr int kEpiWarps = 8;
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kScanThreads = 320;
constexpr int kMaxRows = 64;          // rows per work item
constexpr int kMaxItemCols = 512;     // rows x heads per item
constexpr int kBarEpi = 1;            // named barrier among the epilogue warps

template <MmaKind KIND>
struct ScanCfg {
  static constexpr int ESZ = KIND == MmaKind::TF32 ? 4 : (KIND == MmaKind::BF16 ? 2 : 1);
  static constexpr int A = 128 * ESZ / 128;   // 128-byte atoms per key row (d = 128)
  static constexpr int EPA = 128 / ESZ;       // elements per atom
  static constexpr int KSTAGES = KIND == MmaKind::E4M3 ? 4 : 2;
  static constexpr int KTILE_BYTES = A * 128 * 128;
};

struct ScanSmemTail {
  uint64_t k_full[8], k_empty[8];
  uint64_t q_full, q_empty;
  uint64_t t_full[2], t_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int32_t abort;
  int32_t epi_stop[2];
  int32_t row_cnt[kMaxRows];
  int32_t row_buf[kMaxRows];
  int32_t row_pos[kMaxRows];   // causal position (-1: row absent)
  unsigned long long row_thr[kMaxRows];
  alignas(16) float wsm[kMaxItemCols];
  SelectScratch sel;
};

struct ItemGeom {
  int b, qt, c, row0, nrows, kbeg, kend, ntiles, t_hi;
};

__device__ __forceinline__ ItemGeom item_geom(const ScanArgs& a, int item) {
  ItemGeom g;
  const int per_b = a.n_qt * a.C;
  const int qt_rev = item / (a.batch * a.C);
  const int rem = item % (a.batch * a.C);
  g.b = rem / a.C;
  g.c = rem % a.C;
  g.qt = a.n_qt - 1 - qt_rev;
  (void)per_b;
  const int QT = a.QG * a.G;
  g.row0 = g.qt * QT;
  g.nrows = min(QT, a.n_q - g.row0);
  const int pos0 = a.q_pos0 ? a.q_pos0[g.b] : a.n_k - a.n_q;
  const int klen = a.k_len ? a.k_len[g.b] : a.n_k;
  const int maxpos = pos0 + g.row0 + g.nrows - 1;
  int kend = min(maxpos + 1, klen);
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

template <MmaKind KIND, bool SPLIT>
__global__ void __launch_bounds__(kScanThreads, 1)
    scan_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                const ScanArgs a) {
  using Cfg = ScanCfg<KIND>;
  constexpr int PARTS = SPLIT ? 2 : 1;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int qcols = a.QG * a.H * PARTS;                     // MMA N per group
  uint8_t* Qs = smem;                                       // [G][A][qcols x 128B]
  const int q_bytes = a.G * Cfg::A * qcols * 128;
  uint8_t* Ks = smem + ((q_bytes + 1023) & ~1023);          // [KSTAGES][A][128 x 128B]
  ScanSmemTail* T = reinterpret_cast<ScanSmemTail*>(Ks + Cfg::KSTAGES * Cfg::KTILE_BYTES);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool modeB = (a.QG == 1);  // one query per group: halves take alternate stages

  if (threadIdx.x == 0) {
    for (int i = 0; i < Cfg::KSTAGES; ++i) {
      mbar_init(&T->k_full[i], 1);
      mbar_init(&T->k_empty[i], 1);
    }
    mbar_init(&T->q_full, 1);
    mbar_init(&T->q_empty, 1);
    mbar_init(&T->drain, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&T->t_full[s], 1);
      mbar_init(&T->t_empty[s], modeB ? 4 : 8);
    }
    T->abort = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&T->tmem_base, 2 * a.stage_cols);
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
  const int QT = a.QG * a.G;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer --
    if (lane == 0) {
      uint32_t kcount = 0, it = 0;
      bool ok = true;
      for (int round = 0; ok; ++round) {
        const int item = sched_item(round, blockIdx.x, grid);
        if (item >= a.n_items) break;
        ItemGeom g = item_geom(a, item);
        if (g.ntiles == 0) continue;
        if (!mbar_wait(&T->q_empty, (it & 1) ^ 1, abort, a.status, 1)) break;
        mbar_arrive_expect_tx(&T->q_full, q_bytes);
        const int qrow0 = (g.b * a.n_q + g.row0) * a.H * PARTS;
        for (int gg = 0; gg < a.G; ++gg)
          for (int at = 0; at < Cfg::A; ++at)
            tma_load_2d(Qs + (gg * Cfg::A + at) * qcols * 128, &qmap, &T->q_full,
                        at * Cfg::EPA, qrow0 + gg * a.QG * a.H * PARTS);
        ++it;
        const int krow0 = g.b * a.n_k;
        for (int t = 0; t < g.ntiles && ok; ++t) {
          const int slot = kcount % Cfg::KSTAGES;
          const uint32_t ph = (kcount / Cfg::KSTAGES) & 1;
          if (!mbar_wait(&T->k_empty[slot], ph ^ 1, abort, a.status, 2)) { ok = false; break; }
          mbar_arrive_expect_tx(&T->k_full[slot], Cfg::KTILE_BYTES);
          const int tstart = (g.t_hi - t) << 7;
          for (int at = 0; at < Cfg::A; ++at)
            tma_load_2d(Ks + (slot * Cfg::A + at) * 16384, &kmap, &T->k_full[slot], at * Cfg::EPA,
                        krow0 + tstart);
          ++kcount;
        }
      }
      if (*abort) {
        // abort path: let this CTA's own copies in flight land before exit
        if (it > 0) mbar_wait_drain(&T->q_full, (it - 1) & 1);
        for (uint32_t i = kcount > Cfg::KSTAGES ? kcount - Cfg::KSTAGES : 0; i < kcount; ++i)
          mbar_wait_drain(&T->k_full[i % Cfg::KSTAGES], (i / Cfg::KSTAGES) & 1);
      }
    }
  } else if (warp == kMmaWarp) {
    // ----------------------------------------------------------------- MMA --
    if (lane == 0) {
      const uint32_t idesc = make_idesc<KIND>(qcols);
      uint32_t kcount = 0, ucount = 0, it = 0;
      bool ok = true;
      for (int round = 0; ok; ++round) {
        const int item = sched_item(round, blockIdx.x, grid);
        if (item >= a.n_items) break;
        ItemGeom g = item_geom(a, item);
        if (g.ntiles == 0) continue;
        if (!mbar_wait(&T->q_full, it & 1, abort, a.status, 3)) break;
        ++it;
        tc_fence_after();
        const int nunits = g.ntiles * a.G;
        for (int u = 0; u < nunits; ++u) {
          const int gg = u % a.G;
          const int slot = kcount % Cfg::KSTAGES;
          if (gg == 0) {
            if (!mbar_wait(&T->k_full[slot], (kcount / Cfg::KSTAGES) & 1, abort, a.status, 4)) { ok = false; break; }
          }
          const int s = ucount & 1;
          if (!mbar_wait(&T->t_empty[s], ((ucount >> 1) & 1) ^ 1, abort, a.status, 5)) { ok = false; break; }
          tc_fence_after();
          const uint32_t d = tmem_base + s * a.stage_cols;
          const uint32_t kbase = smem_u32(Ks + slot * Cfg::A * 16384);
          const uint32_t qbase = smem_u32(Qs + gg * Cfg::A * qcols * 128);
#pragma unroll
          for (int at = 0; at < Cfg::A; ++at) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t ad = make_sdesc(kbase + at * 16384 + kk * 32);
              const uint64_t bd = make_sdesc(qbase + at * qcols * 128 + kk * 32);
              tc_mma<KIND>(d, ad, bd, idesc, (at | kk) != 0);
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
        mbar_wait_drain(&T->drain, 0);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue --
    const int etid = threadIdx.x;              // 0..255
    const int quad = warp & 3;                 // TMEM lane quadrant
    const int half = warp >> 2;                // column half / stage (mode B)
    const int H = a.H;
    uint32_t ucount = 0;
    int step_par = 0;
    bool stop = false;
    for (int round = 0; !stop; ++round) {
      const int item = sched_item(round, blockIdx.x, grid);
      if (item >= a.n_items) break;
      ItemGeom g = item_geom(a, item);
      const int pos0 = a.q_pos0 ? a.q_pos0[g.b] : a.n_k - a.n_q;
      const int klen = a.k_len ? a.k_len[g.b] : a.n_k;
      // ---- item init: row states and head weights
      for (int r = etid; r < QT; r += kEpiThreads) {
        T->row_cnt[r] = 0;
        T->row_buf[r] = 0;
        T->row_thr[r] = 0ull;
        T->row_pos[r] = (r < g.nrows) ? pos0 + g.row0 + r : -1;
      }
      for (int i = etid; i < QT * H; i += kEpiThreads) {
        const int r = i / H, j = i % H;
        float wv = 0.f;
        if (r < g.nrows) {
          const int64_t grow = (int64_t)g.b * a.n_q + g.row0 + r;
          wv = a.w[grow * H + j];
          if (a.row_scale) wv *= a.row_scale[grow];
          if (a.head_scale) wv *= a.head_scale[grow * H + j];
        }
        T->wsm[i] = wv;
      }
      named_bar_sync(kBarEpi, kEpiThreads);
      const int nunits = g.ntiles * a.G;
      int u = 0;
      while (u < nunits) {
        // one step = up to two units (stage 0 / stage 1)
        const int nstep = min(2, nunits - u);
        for (int v = 0; v < nstep; ++v) {
          const int uu = u + v;
          const uint32_t uc = ucount + v;
          const int s = uc & 1;
          const bool mine = modeB ? (half == s) : true;
          if (!mine) continue;
          const bool got = mbar_wait(&T->t_full[s], (uc >> 1) & 1, abort, a.status, 6);
          __syncwarp();
          if (!__all_sync(0xffffffffu, got)) continue;
          tc_fence_after();
          const int gg = uu % a.G;
          const int t = uu / a.G;
          const int key = ((g.t_hi - t) << 7) + quad * 32 + lane;
          float ks = 1.f;
          if (a.k_scale && key < a.n_k) ks = a.k_scale[(int64_t)g.b * a.n_k + key];
          const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16) + s * a.stage_cols;
          // queries handled by this warp inside group gg
          const int qbeg = modeB ? 0 : half * (a.QG >> 1);
          const int qnum = modeB ? 1 : (a.QG >> 1);
          const int rbase = gg * a.QG + qbeg;          // first item row of this warp
          // legality, composite key, threshold filter, append (one query row)
          auto finish = [&](int r, float score) {
            score *= ks;
            const int pos = T->row_pos[r];
            const bool legal = pos >= 0 && key <= pos && key < klen && key >= g.kbeg && key < g.kend;
            const uint64_t comp = make_comp(score, key);
            const bool surv = legal && comp >= T->row_thr[r];
            const unsigned bal = __ballot_sync(0xffffffffu, surv);
            if (bal) {
              int base = 0;
              const int leader = __ffs(bal) - 1;
              if (lane == leader) base = atomicAdd(&T->row_cnt[r], __popc(bal));
              base = __shfl_sync(0xffffffffu, base, leader);
              if (surv) {
                const int slot = base + __popc(bal & ((1u << lane) - 1));
                const int64_t rs = ((int64_t)g.b * a.n_q + g.row0 + r) * a.C + g.c;
                a.logs[(rs * 2 + T->row_buf[r]) * a.cap + slot] = comp;
              }
            }
          };
          if (H >= 32) {
            for (int qi = 0; qi < qnum; ++qi) {
              const int r = rbase + qi;
              const float* wr = &T->wsm[r * H];
              const uint32_t cb = taddr + (qbeg + qi) * H * PARTS;
              float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
              for (int c0 = 0; c0 < H; c0 += 32) {
                uint32_t v0[32];
                tmem_ld32(cb + c0, v0);
                if constexpr (SPLIT) {
                  uint32_t v1[32];
                  tmem_ld32(cb + H + c0, v1);
                  tmem_ld_wait();
#pragma unroll
                  for (int jj = 0; jj < 32; jj += 4) {
                    const float4 wv = *reinterpret_cast<const float4*>(wr + c0 + jj);
                    acc0 = fmaf(wv.x, fmaxf(fmaf(__uint_as_float(v1[jj + 0]), 0.0625f, __uint_as_float(v0[jj + 0])), 0.f), acc0);
                    acc1 = fmaf(wv.y, fmaxf(fmaf(__uint_as_float(v1[jj + 1]), 0.0625f, __uint_as_float(v0[jj + 1])), 0.f), acc1);
                    acc2 = fmaf(wv.z, fmaxf(fmaf(__uint_as_float(v1[jj + 2]), 0.0625f, __uint_as_float(v0[jj + 2])), 0.f), acc2);
                    acc3 = fmaf(wv.w, fmaxf(fmaf(__uint_as_float(v1[jj + 3]), 0.0625f, __uint_as_float(v0[jj + 3])), 0.f), acc3);
                  }
                } else {
                  tmem_ld_wait();
#pragma unroll
                  for (int jj = 0; jj < 32; jj += 4) {
                    const float4 wv = *reinterpret_cast<const float4*>(wr + c0 + jj);
                    acc0 = fmaf(wv.x, fmaxf(__uint_as_float(v0[jj + 0]), 0.f), acc0);
                    acc1 = fmaf(wv.y, fmaxf(__uint_as_float(v0[jj + 1]), 0.f), acc1);
                    acc2 = fmaf(wv.z, fmaxf(__uint_as_float(v0[jj + 2]), 0.f), acc2);
                    acc3 = fmaf(wv.w, fmaxf(__uint_as_float(v0[jj + 3]), 0.f), acc3);
                  }
                }
              }
              finish(r, (acc0 + acc1) + (acc2 + acc3));
            }
          } else if constexpr (!SPLIT) {
            // H in {8, 16}: a 32-column load covers 32 / H query rows
            const int ncol = qnum * H;                  // multiple of 32
            for (int c = 0; c < ncol; c += 32) {
              uint32_t v0[32];
              tmem_ld32(taddr + qbeg * H + c, v0);
              tmem_ld_wait();
              const float* wr = &T->wsm[rbase * H + c];
              const int r0 = rbase + c / H;
              if (H == 16) {
#pragma unroll
                for (int qq = 0; qq < 2; ++qq) {
                  float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
#pragma unroll
                  for (int jj = 0; jj < 16; jj += 4) {
                    const float4 wv = *reinterpret_cast<const float4*>(wr + qq * 16 + jj);
                    acc0 = fmaf(wv.x, fmaxf(__uint_as_float(v0[qq * 16 + jj + 0]), 0.f), acc0);
                    acc1 = fmaf(wv.y, fmaxf(__uint_as_float(v0[qq * 16 + jj + 1]), 0.f), acc1);
                    acc2 = fmaf(wv.z, fmaxf(__uint_as_float(v0[qq * 16 + jj + 2]), 0.f), acc2);
                    acc3 = fmaf(wv.w, fmaxf(__uint_as_float(v0[qq * 16 + jj + 3]), 0.f), acc3);
                  }
                  finish(r0 + qq, (acc0 + acc1) + (acc2 + acc3));
                }
              } else {
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) {
                  float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
#pragma unroll
                  for (int jj = 0; jj < 8; jj += 4) {
                    const float4 wv = *reinterpret_cast<const float4*>(wr + qq * 8 + jj);
                    acc0 = fmaf(wv.x, fmaxf(__uint_as_float(v0[qq * 8 + jj + 0]), 0.f), acc0);
                    acc1 = fmaf(wv.y, fmaxf(__uint_as_float(v0[qq * 8 + jj + 1]), 0.f), acc1);
                    acc2 = fmaf(wv.z, fmaxf(__uint_as_float(v0[qq * 8 + jj + 2]), 0.f), acc2);
                    acc3 = fmaf(wv.w, fmaxf(__uint_as_float(v0[qq * 8 + jj + 3]), 0.f), acc3);
                  }
                  finish(r0 + qq, (acc0 + acc1) + (acc2 + acc3));
                }
              }
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&T->t_empty[s]);
        }
        ucount += nstep;
        u += nstep;
        // uniform stop decision: thread 0 snapshots the abort flag before the barrier
        if (etid == 0) T->epi_stop[step_par] = *abort;
        named_bar_sync(kBarEpi, kEpiThreads);
        stop = T->epi_stop[step_par] != 0;
        step_par ^= 1;
        if (stop) break;
        // ---- exact threshold raises for rows whose log is nearly full
        for (int r = 0; r < g.nrows; ++r) {
          if (T->row_cnt[r] <= a.cap - 256) continue;
          const int64_t rs = ((int64_t)g.b * a.n_q + g.row0 + r) * a.C + g.c;
          const int cur = T->row_buf[r];
          const uint64_t* src = a.logs + (rs * 2 + cur) * a.cap;
          uint64_t* dst = a.logs + (rs * 2 + (cur ^ 1)) * a.cap;
          const int n = T->row_cnt[r];
          const uint64_t pfx = radix_select<kEpiThreads>(&src, &n, 1, a.keep, &T->sel, etid, kBarEpi);
          uint64_t kmin;
          const int kept = compact_ge<kEpiThreads>(&src, &n, 1, pfx, dst, &T->sel, etid, kBarEpi, &kmin);
          if (etid == 0) {
            T->row_cnt[r] = kept;
            T->row_buf[r] = cur ^ 1;
            T->row_thr[r] = kmin + 1;
          }
          named_bar_sync(kBarEpi, kEpiThreads);
        }
      }
      // ---- item end: publish log state of every row
      for (int r = etid; r < g.nrows; r += kEpiThreads) {
        const int64_t rs = ((int64_t)g.b * a.n_q + g.row0 + r) * a.C + g.c;
        a.log_cnt[rs] = T->row_cnt[r];
        a.log_buf[rs] = T->row_buf[r];
      }
      if (etid == 0) T->epi_stop[step_par] = *abort;
      named_bar_sync(kBarEpi, kEpiThreads);
      stop = stop || T->epi_stop[step_par] != 0;
      step_par ^= 1;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 2 * a.stage_cols);
  }
}

}  // namespace dsa

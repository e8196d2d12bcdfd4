// finalize.cuh — exact token top-k of each query row from its candidate logs.
//
// The scan leaves, per row and key chunk, a log of composite keys that is a
// superset of the row's top-`keep` keys within that chunk.  This kernel takes
// the exact top-k over all the row's logs (radix select on the composite key,
// so a lower token index wins a score tie), orders the winners by
// (score descending, index ascending) and writes int32 indices + fp32 scores,
// padding with (-1, -inf) when the row has fewer than k legal keys — the output
// contract of the indexer's token top-k ("PaperTrace 2.2.2 MISA, LISA and
// ResMiSA", section 2.2: score, causal mask and top-k feed Sparse MLA as
// integer positions; section 2.3: stable ordering on ties).
#pragma once
#include "common.cuh"
#include "select.cuh"

namespace dsa {

constexpr int kFinMaxGroups = 4;       // row groups per CTA
constexpr int kFinMaxSeg = 128;

struct FinalArgs {
  int32_t rows;
  int32_t C;             // key chunks per row
  int32_t nsub;          // sub-logs per (row, chunk) slot
  int32_t topk;
  int32_t capw;          // entries per sub-log
  int32_t sort_cap;      // power of two >= topk
  int32_t sorted;        // 1: order by (score desc, index asc); 2: by index asc; 0: any order
  const uint64_t* logs;  // [rows * C][nsub][capw]
  const int32_t* log_cnt;               // [rows * C][nsub]
  const unsigned long long* log_thr;    // [rows * C]
  int32_t nq_c;          // rows per sequence in this call (rows = batch * nq_c)
  int32_t nq_total;      // rows per sequence of the outputs
  int32_t q_off;         // row i of sequence b writes output row b * nq_total + q_off + i
  int32_t* out_idx;      // [batch * nq_total, topk]
  float* out_score;      // [batch * nq_total, topk] or null
  const int32_t* status; // workspace status word: a failed scan leaves its logs
                         //   unfinished, and the rows are then written as padding
};

constexpr int kFinBoundary = 1024;  // boundary-bin capacity per row group

// Per-row-group scalars.
struct FinGroup {
  SelectScratch sc;
  int staged, nwin, nbnd, fallback;
  unsigned long long thr;
};

// Shared memory of one row group: [sort_cap] result keys, [stage_cap] staged
// candidates, [kFinBoundary] boundary-bin candidates.  NT threads per row
// group: 256 when a row has one key chunk (about k candidates), 1024 for
// split-K rows (about C * k candidates).  E = sort_cap / NT keys per thread
// for the optional ordering.
//
// Selection.  thr, the largest of the row's slot thresholds, bounds the row's
// k-th best from below.  Candidates >= thr are staged and counted in 256 bins
// of 16-bit score-key resolution above thr; the bin b* holding the k-th best
// is found from the counts, every candidate in a higher bin is a winner, and
// the (small) boundary bin b* is ranked exactly by one warp.  A boundary bin
// too large for that, or a k-th best beyond the bin window, falls back to the
// radix select.
template <int NT, int E>
__global__ void __launch_bounds__(E <= 8 ? 1024 : NT)
    finalize_kernel(const FinalArgs a, int groups, int stage_cap) {
  extern __shared__ __align__(16) uint64_t fin_smem[];
  __shared__ FinGroup fg_all[kFinMaxGroups];
  __shared__ const uint64_t* segp_all[kFinMaxGroups][kFinMaxSeg];
  __shared__ int segn_all[kFinMaxGroups][kFinMaxSeg];
  __shared__ unsigned long long segt_all[kFinMaxGroups][kFinMaxSeg];
  const int grp = threadIdx.x / NT;
  const int tid = threadIdx.x % NT;
  const int lane = tid & 31;
  const int bar = 1 + grp;
  const int row = blockIdx.x * groups + grp;
  if (grp >= groups || row >= a.rows) return;   // whole groups leave together
  uint64_t* out = fin_smem + (size_t)grp * (a.sort_cap + stage_cap + kFinBoundary);
  uint64_t* stage = out + a.sort_cap;
  uint64_t* bnd = stage + stage_cap;
  FinGroup* G = &fg_all[grp];
  const uint64_t** segp = segp_all[grp];
  int* segn = segn_all[grp];
  unsigned long long* segt = segt_all[grp];
  const int nseg = a.C * a.nsub;
  // after a device error (a scan that gave up on a wait) the logs and their
  // fills are not this call's: read none of them, write the padding
  const bool failed = *reinterpret_cast<const volatile int32_t*>(a.status) != DSA_OK;
  for (int g = tid; g < nseg; g += NT) {
    const int c = g / a.nsub, sb = g % a.nsub;
    const int64_t rs = (int64_t)row * a.C + c;
    segp[g] = a.logs + (rs * a.nsub + sb) * a.capw;
    const int n = failed ? 0 : a.log_cnt[rs * a.nsub + sb];
    segn[g] = n < 0 ? 0 : (n > a.capw ? a.capw : n);
    segt[g] = failed ? 0ull : a.log_thr[rs];
  }
  for (int i = tid; i < 256; i += NT) G->sc.hist[i] = 0;
  if (tid == 0) {
    G->staged = G->nwin = G->nbnd = G->fallback = 0;
    G->thr = 0ull;
  }
  named_bar_sync(bar, NT);
  if (tid == 0) {
    unsigned long long t = 0ull;
    for (int g = 0; g < a.C; ++g) t = segt[g * a.nsub] > t ? segt[g * a.nsub] : t;
    G->thr = t;
  }
  named_bar_sync(bar, NT);
  const unsigned long long thr = G->thr;
  const int thr16 = (int)(thr >> 48);
  // ---- stage candidates >= thr and count them per 16-bit score-key bin above
  // thr; segments are spread over the group's warps, eight loads per lane in flight
  constexpr int NW = NT / 32;
  const int wid = tid >> 5;
  // fewer segments than warps: several warps share a segment (parts of 256)
  const int parts = nseg >= NW ? 1 : NW / nseg;
  const int g0 = nseg >= NW ? wid : (wid < parts * nseg ? wid % nseg : nseg);
  const int gstep = nseg >= NW ? NW : nseg;
  const int part = nseg >= NW ? 0 : wid / nseg;
  // every candidate >= thr of the row's logs, warp-uniformly: fn(v, is_candidate)
  auto for_each_candidate = [&](auto&& fn) {
    for (int g = g0; g < nseg; g += gstep) {
      const uint64_t* p = segp[g];
      const int n = segn[g];
      for (int i0 = part * 256; i0 < n; i0 += parts * 256) {
        uint64_t v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int i = i0 + j * 32 + lane;
          v[j] = i < n ? p[i] : 0ull;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) fn(v[j], i0 + j * 32 + lane < n && v[j] >= thr);
      }
    }
  };
  for_each_candidate([&](uint64_t v, bool keep) {
    const unsigned bal = __ballot_sync(0xffffffffu, keep);
    if (bal) {
      int base = 0;
      if (lane == 0) base = atomicAdd(&G->staged, __popc(bal));
      base = __shfl_sync(0xffffffffu, base, 0);
      if (keep) {
        const int slot = base + __popc(bal & ((1u << lane) - 1));
        if (slot < stage_cap) stage[slot] = v;
        atomicAdd(&G->sc.hist[min(255, (int)(v >> 48) - thr16)], 1);
      }
    }
  });
  named_bar_sync(bar, NT);
  const int total = G->staged;
  int n;  // number of result keys in out[]
  if (total <= stage_cap && total <= a.topk) {
    // every candidate is a winner
    for (int i = tid; i < total; i += NT) out[i] = stage[i];
    n = total;
  } else {
    // more candidates than the stage holds: the histogram is still complete, so
    // winners and the boundary bin are taken from the logs in a second read
    const bool overflow = total > stage_cap;
    bool fb = false;
    int bstar = 0, above = 0;
    // the 256 bins cover score-key prefixes base16 .. base16 + 254 (bin 255 holds
    // everything higher); a k-th best beyond that window moves the window up and
    // recounts (the candidates below the new base cannot be among the top k)
    int base16 = thr16;
    for (int window = 0;; ++window) {
      if (tid < 32) {
        int ab;
        const int b = hist_find(reinterpret_cast<const uint32_t*>(G->sc.hist), 0, a.topk, lane, &ab);
        if (lane == 0) {
          G->sc.sel[0] = b;
          G->sc.sel[1] = ab;
          G->fallback = (b < 0 || (b == 255 && window == 7)) ? 1 : 0;
        }
      }
      named_bar_sync(bar, NT);
      fb = G->fallback != 0;
      bstar = G->sc.sel[0];
      above = G->sc.sel[1];
      if (fb || bstar < 255) break;
      base16 += 255;
      for (int i = tid; i < 256; i += NT) G->sc.hist[i] = 0;
      named_bar_sync(bar, NT);
      auto recount = [&](uint64_t v, bool cand) {
        const int bin = cand ? min(255, (int)(v >> 48) - base16) : -1;
        if (bin >= 0) atomicAdd(&G->sc.hist[bin], 1);
      };
      if (!overflow) {
        for (int i = tid; i < total; i += NT) recount(stage[i], true);
      } else {
        for_each_candidate(recount);
      }
      named_bar_sync(bar, NT);
    }
    if (!fb) {
      // winners above the boundary bin; the boundary bin's candidates aside
      auto sort_out = [&](uint64_t v, bool cand) {
        const int bin = cand ? min(255, (int)(v >> 48) - base16) : -1;
        const bool win = bin > bstar, edge = bin == bstar;
        const unsigned bw = __ballot_sync(0xffffffffu, win);
        const unsigned be = __ballot_sync(0xffffffffu, edge);
        int bwin = 0, bedge = 0;
        if (lane == 0) {
          if (bw) bwin = atomicAdd(&G->nwin, __popc(bw));
          if (be) bedge = atomicAdd(&G->nbnd, __popc(be));
        }
        bwin = __shfl_sync(0xffffffffu, bwin, 0);
        bedge = __shfl_sync(0xffffffffu, bedge, 0);
        const unsigned lt = (1u << lane) - 1;
        if (win) out[bwin + __popc(bw & lt)] = v;
        if (edge) {
          const int slot = bedge + __popc(be & lt);
          if (slot < kFinBoundary) bnd[slot] = v;
        }
      };
      if (!overflow) {
        for (int i0 = 0; i0 < total; i0 += NT) {
          const int i = i0 + tid;
          sort_out(i < total ? stage[i] : 0ull, i < total);
        }
      } else {
        for_each_candidate(sort_out);
      }
      named_bar_sync(bar, NT);
      const int nb = G->nbnd;
      const int need = a.topk - above;
      if (nb <= 256) {
        if (tid < 32) warp_take_top(bnd, nb, need, out, above, lane);
        named_bar_sync(bar, NT);
        n = a.topk;
      } else if (nb <= kFinBoundary) {
        const uint64_t* bs[1] = {bnd};
        const int bn[1] = {nb};
        const uint64_t t2 = radix_select<NT>(bs, bn, 1, need, &G->sc, tid, bar);
        // append the boundary keys >= t2 after the winners
        if (tid == 0) G->sc.newcnt = 0;
        named_bar_sync(bar, NT);
        for (int i = tid; i < nb; i += NT)
          if (bnd[i] >= t2) out[above + atomicAdd(&G->sc.newcnt, 1)] = bnd[i];
        named_bar_sync(bar, NT);
        n = a.topk;
      } else {
        fb = true;
      }
    }
    if (fb) {
      // generic exact selection (long runs of ties): radix select over the
      // staged set when it fits, else over the raw logs
      const uint64_t* one[1] = {stage};
      const int one_n[1] = {total};
      const bool staged_ok = total <= stage_cap;
      const uint64_t* const* sp = staged_ok ? one : segp;
      const int* sn = staged_ok ? one_n : segn;
      const int ns = staged_ok ? 1 : nseg;
      const uint64_t t = radix_select<NT>(sp, sn, ns, a.topk, &G->sc, tid, bar);
      n = compact_ge<NT>(sp, sn, ns, t, out, &G->sc, tid, bar, nullptr);
    }
  }
  if (a.sorted == 2) {
    // position order: sort on (~index, score) — the composite with its halves
    // swapped — descending, which is index ascending (indices are unique)
    named_bar_sync(bar, NT);
    for (int i = tid; i < n; i += NT) out[i] = (out[i] << 32) | (out[i] >> 32);
    sort_desc_regs<NT, E>(out, n, tid, bar);
    for (int i = tid; i < n; i += NT) out[i] = (out[i] << 32) | (out[i] >> 32);
    named_bar_sync(bar, NT);
  } else if (a.sorted) {
    sort_desc_regs<NT, E>(out, n, tid, bar);   // sort_cap == NT * E
  }
  const int64_t orow = (int64_t)(row / a.nq_c) * a.nq_total + a.q_off + row % a.nq_c;
  int32_t* oi = a.out_idx + orow * a.topk;
  float* os = a.out_score ? a.out_score + orow * a.topk : nullptr;
  for (int i = tid; i < a.topk; i += NT) {
    if (i < n) {
      const uint64_t c = out[i];
      oi[i] = comp_index(c);
      if (os) os[i] = comp_score(c);
    } else {
      oi[i] = -1;
      if (os) os[i] = -__int_as_float(0x7f800000);
    }
  }
}

}  // namespace dsa

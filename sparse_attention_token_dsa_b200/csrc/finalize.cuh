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

constexpr int kFinGroupThreads = 256;  // threads per row group (one named barrier each)
constexpr int kFinMaxGroups = 4;       // row groups per CTA
constexpr int kFinMaxSeg = 128;

struct FinalArgs {
  int32_t rows;
  int32_t C;             // key chunks per row
  int32_t nsub;          // sub-logs per (row, chunk) slot
  int32_t topk;
  int32_t capw;          // entries per sub-log
  int32_t sort_cap;      // power of two >= topk
  int32_t sorted;        // 1: order by (score desc, index asc); 0: any order
  const uint64_t* logs;  // [rows * C][nsub][capw]
  const int32_t* log_cnt;               // [rows * C][nsub]
  const unsigned long long* log_thr;    // [rows * C]
  int32_t* out_idx;      // [rows, topk]
  float* out_score;      // [rows, topk] or null
};

// Shared memory of one row group: [sort_cap] selected keys, then [stage_cap]
// staged candidates.  NT threads per row group: 256 when a row has one key
// chunk (about k candidates), 1024 for split-K rows (about C * k candidates).
template <int NT>
__global__ void __launch_bounds__(1024)
    finalize_kernel(const FinalArgs a, int groups, int stage_cap) {
  constexpr int kFinGroupThreads = NT;
  extern __shared__ __align__(16) uint64_t fin_smem[];
  __shared__ SelectScratch sc_all[kFinMaxGroups];
  __shared__ const uint64_t* segp_all[kFinMaxGroups][kFinMaxSeg];
  __shared__ int segn_all[kFinMaxGroups][kFinMaxSeg];
  __shared__ unsigned long long segt_all[kFinMaxGroups][kFinMaxSeg];
  __shared__ int staged_all[kFinMaxGroups];
  const int grp = threadIdx.x / kFinGroupThreads;
  const int tid = threadIdx.x % kFinGroupThreads;
  const int bar = 1 + grp;
  const int row = blockIdx.x * groups + grp;
  if (grp >= groups || row >= a.rows) return;   // whole groups leave together
  uint64_t* fin_buf = fin_smem + (size_t)grp * (a.sort_cap + stage_cap);
  uint64_t* stage = fin_buf + a.sort_cap;
  SelectScratch* sc = &sc_all[grp];
  const uint64_t** segp = segp_all[grp];
  int* segn = segn_all[grp];
  unsigned long long* segt = segt_all[grp];
  const int nseg = a.C * a.nsub;
  for (int g = tid; g < nseg; g += kFinGroupThreads) {
    const int c = g / a.nsub, sb = g % a.nsub;
    const int64_t rs = (int64_t)row * a.C + c;
    segp[g] = a.logs + (rs * a.nsub + sb) * a.capw;
    segn[g] = a.log_cnt[rs * a.nsub + sb];
    segt[g] = a.log_thr[rs];
  }
  if (tid == 0) staged_all[grp] = 0;
  named_bar_sync(bar, kFinGroupThreads);
  // stage the candidates at or above their slot's threshold (a superset of the
  // row's top-k: each slot's threshold bounds that slot's own top-k from below)
  // eight independent loads per thread in flight; one slot reservation per warp
  const int lane = tid & 31;
  for (int g = 0; g < nseg; ++g) {
    const uint64_t* p = segp[g];
    const int n = segn[g];
    const unsigned long long t = segt[g];
    for (int i0 = 0; i0 < n; i0 += 8 * kFinGroupThreads) {
      uint64_t v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int i = i0 + j * kFinGroupThreads + tid;
        v[j] = i < n ? p[i] : 0ull;
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int i = i0 + j * kFinGroupThreads + tid;
        const bool keep = i < n && v[j] >= t;
        const unsigned bal = __ballot_sync(0xffffffffu, keep);
        if (bal) {
          int base = 0;
          if (lane == 0) base = atomicAdd(&staged_all[grp], __popc(bal));
          base = __shfl_sync(0xffffffffu, base, 0);
          const int slot = base + __popc(bal & ((1u << lane) - 1));
          if (keep && slot < stage_cap) stage[slot] = v[j];
        }
      }
    }
  }
  named_bar_sync(bar, kFinGroupThreads);
  const int total = staged_all[grp];
  const uint64_t* one[1];
  int one_n[1];
  const uint64_t* const* sp;
  const int* sn;
  int ns;
  bool staged = total <= stage_cap;
  if (staged) {
    one[0] = stage;
    one_n[0] = total;
    sp = one;
    sn = one_n;
    ns = 1;
  } else {  // too many to stage (long runs of tied scores): select from the logs
    sp = segp;
    sn = segn;
    ns = nseg;
  }
  uint64_t thr = 0ull;
  if (!staged || total > a.topk)
    thr = radix_select<kFinGroupThreads>(sp, sn, ns, a.topk, sc, tid, bar);
  const int n = compact_ge<kFinGroupThreads>(sp, sn, ns, thr, fin_buf, sc, tid, bar, nullptr);
  if (a.sorted) bitonic_sort_desc<kFinGroupThreads>(fin_buf, n, a.sort_cap, tid, bar);
  int32_t* oi = a.out_idx + (int64_t)row * a.topk;
  float* os = a.out_score ? a.out_score + (int64_t)row * a.topk : nullptr;
  for (int i = tid; i < a.topk; i += kFinGroupThreads) {
    if (i < n) {
      const uint64_t c = fin_buf[i];
      oi[i] = comp_index(c);
      if (os) os[i] = comp_score(c);
    } else {
      oi[i] = -1;
      if (os) os[i] = -__int_as_float(0x7f800000);
    }
  }
}

}  // namespace dsa

// select.cuh — exact block-cooperative selection on 64-bit composite keys.
//
// A composite key packs (order-preserving score bits << 32 | ~index): a larger
// key is a better candidate and a lower token index wins a score tie, which is
// the total order the indexer's top-k uses ("PaperTrace 2.2.2 MISA, LISA and
// ResMiSA", section 2.3 end-to-end acceptance: stable sort, ties resolved
// consistently).  radix_select finds, over one or more key segments, the
// smallest prefix P such that exactly `need` keys are >= P (keys are unique).
#pragma once
#include "common.cuh"

namespace dsa {

struct SelectScratch {
  int hist[256];
  int sel[4];
  unsigned long long kmin;
  int newcnt;
  int pad;
};

// nthr threads with ids [0, nthr) call this together; threads 0..31 must be one
// warp.  bar_id names the barrier the group synchronises on.  Requires that the
// segments hold at least `need` keys in total and need >= 1.
template <int NTHR>
__device__ uint64_t radix_select(const uint64_t* const* seg, const int* seg_n, int nseg, int need,
                                 SelectScratch* sc, int tid, int bar_id) {
  uint64_t prefix = 0, mask = 0;
  for (int shift = 56; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += NTHR) sc->hist[i] = 0;
    named_bar_sync(bar_id, NTHR);
    // histogram of the next digit; lanes sharing a bin add once (one atomic per
    // distinct bin per warp: candidates cluster in very few bins)
    for (int g = 0; g < nseg; ++g) {
      const uint64_t* p = seg[g];
      const int n = seg_n[g];
      for (int i0 = 0; i0 < n; i0 += NTHR) {
        const int i = i0 + tid;
        const uint64_t v = i < n ? p[i] : 0ull;
        const bool m = i < n && (v & mask) == prefix;
        const unsigned act = __ballot_sync(0xffffffffu, m);
        if (m) {
          const int bin = (int)((v >> shift) & 255);
          const unsigned peers = __match_any_sync(act, bin);
          if ((tid & 31) == __ffs(peers) - 1) atomicAdd(&sc->hist[bin], __popc(peers));
        }
      }
    }
    named_bar_sync(bar_id, NTHR);
    if (tid < 32) {
      const int lane = tid;
      int c[8], tot = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        c[i] = sc->hist[255 - 8 * lane - i];
        tot += c[i];
      }
      int incl = tot;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        int o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
      }
      const int excl = incl - tot;
      const bool mine = excl < need && need <= incl;
      const unsigned bal = __ballot_sync(0xffffffffu, mine);
      if (bal != 0 && lane == __ffs(bal) - 1) {
        int cum = excl;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (cum + c[i] >= need) {
            sc->sel[0] = 255 - 8 * lane - i;
            sc->sel[1] = cum;
            sc->sel[2] = c[i];
            break;
          }
          cum += c[i];
        }
      }
    }
    named_bar_sync(bar_id, NTHR);
    const int bin = sc->sel[0], above = sc->sel[1], cnt = sc->sel[2];
    named_bar_sync(bar_id, NTHR);
    need -= above;
    prefix |= (uint64_t)bin << shift;
    mask |= (uint64_t)0xFF << shift;
    if (cnt == need) break;
  }
  return prefix;
}

// Copy the keys >= thr of the segments into out (unordered).  Returns the
// count; *kmin (when not null) receives the smallest copied key (all threads
// see both).
template <int NTHR>
__device__ int compact_ge(const uint64_t* const* seg, const int* seg_n, int nseg, uint64_t thr,
                          uint64_t* out, SelectScratch* sc, int tid, int bar_id, uint64_t* kmin) {
  if (tid == 0) {
    sc->newcnt = 0;
    sc->kmin = ~0ull;
  }
  named_bar_sync(bar_id, NTHR);
  for (int g = 0; g < nseg; ++g) {
    const uint64_t* p = seg[g];
    const int n = seg_n[g];
    for (int i0 = 0; i0 < n; i0 += NTHR) {
      const int i = i0 + tid;
      const uint64_t v = i < n ? p[i] : 0ull;
      const bool keep = i < n && v >= thr;
      const unsigned bal = __ballot_sync(0xffffffffu, keep);
      if (bal) {
        const int lane = tid & 31;
        int base = 0;
        if (lane == 0) base = atomicAdd(&sc->newcnt, __popc(bal));
        base = __shfl_sync(0xffffffffu, base, 0);
        if (keep) out[base + __popc(bal & ((1u << lane) - 1))] = v;
        if (kmin) {  // warp minimum of the kept keys, one atomic per warp
          unsigned long long m = keep ? v : ~0ull;
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) {
            const unsigned long long o = __shfl_xor_sync(0xffffffffu, m, off);
            m = o < m ? o : m;
          }
          if (lane == 0) atomicMin(&sc->kmin, m);
        }
      }
    }
  }
  named_bar_sync(bar_id, NTHR);
  const int n = sc->newcnt;
  if (kmin) *kmin = sc->kmin;
  named_bar_sync(bar_id, NTHR);
  return n;
}

// In-place descending bitonic sort of n <= cap keys in shared memory (cap a
// power of two; slots [n, cap) are filled with 0, the smallest key).
template <int NTHR>
__device__ void bitonic_sort_desc(uint64_t* a, int n, int cap, int tid, int bar_id) {
  for (int i = n + tid; i < cap; i += NTHR) a[i] = 0ull;
  named_bar_sync(bar_id, NTHR);
  for (int size = 2; size <= cap; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = tid; i < cap / 2; i += NTHR) {
        int lo = 2 * i - (i & (stride - 1));
        int hi = lo + stride;
        bool desc = ((lo & size) == 0);
        uint64_t x = a[lo], y = a[hi];
        if ((x < y) == desc) {
          a[lo] = y;
          a[hi] = x;
        }
      }
      named_bar_sync(bar_id, NTHR);
    }
  }
}

}  // namespace dsa

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

// Warp-wide search over 256 histogram bins (lane l owns bins 255-8l .. 248-8l):
// the highest bin b with base + (count of bins >= b) >= need.  Returns the bin
// (-1 when the total stays below need) and, in *above, base + count strictly
// above it.
__device__ __forceinline__ int hist_find(const uint32_t* h, int base, int need, int lane,
                                         int* above) {
  int c[8];
  int tot = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    c[i] = (int)h[255 - 8 * lane - i];
    tot += c[i];
  }
  int incl = tot;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  const int excl = incl - tot;
  const bool mine = base + excl < need && need <= base + incl;
  const unsigned bal = __ballot_sync(0xffffffffu, mine);
  if (!bal) {
    *above = 0;
    return -1;
  }
  const int src = __ffs(bal) - 1;
  int bin = 0, ab = 0;
  if (lane == src) {
    int cum = base + excl;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (cum + c[i] >= need) {
        bin = 255 - 8 * lane - i;
        ab = cum;
        break;
      }
      cum += c[i];
    }
  }
  *above = __shfl_sync(0xffffffffu, ab, src);
  return __shfl_sync(0xffffffffu, bin, src);
}

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

// Descending bitonic sort of N = NT * E keys held E per thread in registers
// (thread t holds positions t*E .. t*E+E-1).  Strides below E compare inside a
// thread, strides below 32*E across lanes with shuffles, and only strides of
// 32*E and more go through shared memory `xs` (N keys) with a barrier.
template <int NT, int E>
__device__ __forceinline__ void bitonic_regs_desc(uint64_t (&v)[E], uint64_t* xs, int tid,
                                                  int bar_id) {
  constexpr int N = NT * E;
  const int lane = tid & 31;
#pragma unroll
  for (int size = 2; size <= N; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      if (stride < E) {
#pragma unroll
        for (int e = 0; e < E; ++e) {
          if ((e & stride) == 0) {
            const int i = tid * E + e;
            const bool desc = (i & size) == 0;
            const uint64_t x = v[e], y = v[e + stride];
            if ((x < y) == desc) {
              v[e] = y;
              v[e + stride] = x;
            }
          }
        }
      } else if (stride < 32 * E) {
        const int ld = stride / E;  // lane distance of the partner
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const int i = tid * E + e;
          const uint64_t o = __shfl_xor_sync(0xffffffffu, v[e], ld);
          const bool lower = (lane & ld) == 0;      // this position is the pair's lower index
          const bool desc = (i & size) == 0;
          // the lower position keeps the larger key in a descending pair
          const bool take_max = lower == desc;
          v[e] = take_max ? (o > v[e] ? o : v[e]) : (o < v[e] ? o : v[e]);
        }
      } else {
#pragma unroll
        for (int e = 0; e < E; ++e) xs[tid * E + e] = v[e];
        named_bar_sync(bar_id, NT);
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const int i = tid * E + e;
          const uint64_t o = xs[i ^ stride];
          const bool lower = (i & stride) == 0;
          const bool desc = (i & size) == 0;
          const bool take_max = lower == desc;
          v[e] = take_max ? (o > v[e] ? o : v[e]) : (o < v[e] ? o : v[e]);
        }
        named_bar_sync(bar_id, NT);
      }
    }
  }
}

// Sort a[0, n) descending in place (n <= N = NT * E; slots up to N hold 0).
// Thread t reads slots written by other threads: the group synchronises first.
template <int NT, int E>
__device__ void sort_desc_regs(uint64_t* a, int n, int tid, int bar_id) {
  named_bar_sync(bar_id, NT);
  uint64_t v[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int i = tid * E + e;
    v[e] = i < n ? a[i] : 0ull;
  }
  named_bar_sync(bar_id, NT);
  bitonic_regs_desc<NT, E>(v, a, tid, bar_id);
#pragma unroll
  for (int e = 0; e < E; ++e) a[tid * E + e] = v[e];
  named_bar_sync(bar_id, NT);
}

// Exact selection of the `need` largest of the n <= 256 distinct keys in b[]
// by one warp, appended to out[base..] in descending order: each key's rank is
// the number of larger keys (n compares per key, read as smem broadcasts).
__device__ __forceinline__ void warp_take_top(const uint64_t* b, int n, int need, uint64_t* out,
                                              int base, int lane) {
  for (int i = lane; i < n; i += 32) {
    const uint64_t v = b[i];
    int rank = 0;
    for (int j = 0; j < n; ++j) rank += b[j] > v ? 1 : 0;
    if (rank < need) out[base + rank] = v;
  }
}

}  // namespace dsa

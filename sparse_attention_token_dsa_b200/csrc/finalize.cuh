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

constexpr int kFinThreads = 512;
constexpr int kFinMaxSeg = 64;

struct FinalArgs {
  int32_t rows;
  int32_t C;             // log segments per row
  int32_t topk;
  int32_t cap;
  int32_t sort_cap;      // power of two >= topk
  int32_t sorted;        // 1: order by (score desc, index asc); 0: any order
  const uint64_t* logs;  // [rows * C][2][cap]
  const int32_t* log_cnt;
  const int32_t* log_buf;
  int32_t* out_idx;      // [rows, topk]
  float* out_score;      // [rows, topk] or null
};

__global__ void __launch_bounds__(kFinThreads) finalize_kernel(const FinalArgs a) {
  extern __shared__ __align__(16) uint64_t fin_buf[];
  __shared__ SelectScratch sc;
  __shared__ const uint64_t* segp[kFinMaxSeg];
  __shared__ int segn[kFinMaxSeg];
  __shared__ int total_s;
  const int row = blockIdx.x;
  const int tid = threadIdx.x;
  if (tid < a.C) {
    const int64_t rs = (int64_t)row * a.C + tid;
    segp[tid] = a.logs + (rs * 2 + a.log_buf[rs]) * a.cap;
    segn[tid] = a.log_cnt[rs];
  }
  __syncthreads();
  if (tid == 0) {
    int t = 0;
    for (int g = 0; g < a.C; ++g) t += segn[g];
    total_s = t;
  }
  __syncthreads();
  const int total = total_s;
  uint64_t thr = 0ull;
  if (total > a.topk) thr = radix_select<kFinThreads>(segp, segn, a.C, a.topk, &sc, tid, 1);
  uint64_t kmin;
  const int n = compact_ge<kFinThreads>(segp, segn, a.C, thr, fin_buf, &sc, tid, 1, &kmin);
  if (a.sorted) bitonic_sort_desc<kFinThreads>(fin_buf, n, a.sort_cap, tid, 1);
  int32_t* oi = a.out_idx + (int64_t)row * a.topk;
  float* os = a.out_score ? a.out_score + (int64_t)row * a.topk : nullptr;
  for (int i = tid; i < a.topk; i += kFinThreads) {
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

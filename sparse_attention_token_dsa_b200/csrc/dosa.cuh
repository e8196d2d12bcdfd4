// dosa.cuh — DoSA block upper bounds of the indexer score, on tcgen05.
//
// "The new bottleneck of sparse attention", route five (DoSA): a candidate
// whose upper bound lies below a lower bound of the k-th best score cannot
// enter the top-k, so its full score need not be formed.  Here the candidates
// are grouped in blocks of 2^shift consecutive keys and bounded through the
// block's per-dimension key range [kmin_c, kmax_c]: over that box,
//     hi_j = max q_j . k = sum_c q+_c kmax_c + q-_c kmin_c
//     lo_j = min q_j . k = sum_c q+_c kmin_c + q-_c kmax_c
// (q+ = max(q, 0), q- = min(q, 0)), and since ReLU is monotone
//     I_{t,s} <= UB_{t,b} = sum_j (w_j > 0 ? w_j ReLU(hi_j) : w_j ReLU(lo_j))
// for every key s of block b.  Both box extremes are one contraction over
// K = 256: A_j = [q+ | q-] against the block rows [kmax | kmin] (hi) and
// [kmin | kmax] (lo), i.e. a GEMM of (rows x heads) x 256 by 256 x (2 x blocks).
//
// Rounding: the tensor-core sums (here over 256 products, in the scan over
// 128), the fp32 weighted head sums of both kernels and this kernel's own
// adds each err by less than 2^-15 |w_j| ||q_j||_1 mx_b, where mx_b is the
// largest |k_c| of the block; UB adds 2^-12 sum_j |w_j| ||q_j||_1 mx_b, so
// it bounds the score exactly as the scan computes it.
//
// The same box gives a lower bound of every key's score in the block,
//     LB_{t,b} = sum_j (w_j > 0 ? w_j ReLU(lo_j) : w_j ReLU(hi_j)) - slack,
// and so the seed set of the pages' DoSA: the blocks of largest LB, taken until
// they hold keep legal keys, guarantee keep keys scoring at least the last
// one's LB — a lower bound of the row's keep-th best score before any key is
// scanned.  The scan starts each row's threshold there, then raises it as it
// goes; it skips the head sums of a (row, key tile) whose block UB lies below
// the threshold.  Every candidate either skipped or filtered out by the seed
// lies below the keep-th best, so the selected set is unchanged.
#pragma once
#include "common.cuh"

namespace dsa {

// ------------------------------------------------------------ key ranges --
// E [batch][2][nblk][256] bf16: E[b][0][blk] = (kmax | kmin), E[b][1][blk] =
// (kmin | kmax); mx [batch][nblk] = max_c max(|kmin_c|, |kmax_c|).  The last
// block of a sequence may be partial (its range covers the keys present).
// bf16 keys: minima, maxima and magnitudes are exact.
__global__ void __launch_bounds__(128)
    dosa_ranges_kernel(const uint16_t* __restrict__ k, int n_tok, int shift, int nblk,
                       uint16_t* __restrict__ E, float* __restrict__ mx) {
  __shared__ float wmax[4];
  const int blk = blockIdx.x, b = blockIdx.y, c = threadIdx.x;
  const int s0 = blk << shift;
  const int s1 = min(s0 + (1 << shift), n_tok);
  float mn = __int_as_float(0x7f800000), mxv = -__int_as_float(0x7f800000);
  for (int sb = s0; sb < s1; sb += 8) {
    float x[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int s = min(sb + e, s1 - 1);
      x[e] = __uint_as_float((uint32_t)k[((int64_t)b * n_tok + s) * 128 + c] << 16);
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      mn = fminf(mn, x[e]);
      mxv = fmaxf(mxv, x[e]);
    }
  }
  const uint16_t lo = (uint16_t)(__float_as_uint(mn) >> 16);
  const uint16_t hi = (uint16_t)(__float_as_uint(mxv) >> 16);
  uint16_t* e0 = E + (((int64_t)b * 2 + 0) * nblk + blk) * 256;
  uint16_t* e1 = E + (((int64_t)b * 2 + 1) * nblk + blk) * 256;
  e0[c] = hi;
  e0[128 + c] = lo;
  e1[c] = lo;
  e1[128 + c] = hi;
  float m = fmaxf(fabsf(mn), fabsf(mxv));
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((c & 31) == 0) wmax[c >> 5] = m;
  __syncthreads();
  if (c == 0) mx[(int64_t)b * nblk + blk] = fmaxf(fmaxf(wmax[0], wmax[1]), fmaxf(wmax[2], wmax[3]));
}

// ------------------------------------------------------------ bound GEMM --
constexpr int kDosaThreads = 192;      // warps 0-3 epilogue, 4 TMA producer, 5 MMA issuer
constexpr int kDosaBT = 32;            // bound blocks per B tile (N = 64: hi and lo rows)
constexpr int kDosaKS = 1;             // B tile buffers (one: two CTAs fit an SM)

struct DosaArgs {
  int32_t batch, n_q, n_tok, H;
  int32_t shift;             // bound block = 2^shift keys
  int32_t nblk;              // blocks per sequence (ceil(n_tok / block))
  const int32_t* q_pos0;     // [batch] or null: n_tok - n_q
  const int32_t* k_len;      // [batch] or null: n_tok
  const float* w;            // [batch * n_q, H]
  const float* mx;           // [batch, nblk]
  float* ub;                 // [batch * n_q, nblk]; blocks past the row's legal keys: -inf
  float* lb;                 // [batch * n_q, nblk] lower bounds (same blocks), or null
  int32_t* status;
};

struct DosaSmemTail {
  uint64_t q_full, a_ready, drain;
  uint64_t e_full[kDosaKS], e_empty[kDosaKS];
  uint64_t d_full[2], d_empty[2];
  uint32_t tmem_base;
  int32_t abort;
  float part[2][4][kDosaBT];  // per-warp head sums of a tile (double-buffered)
  float partl[2][4][kDosaBT]; // the same for the lower bounds
  int32_t okw[2][4];          // the warp's round completed (its partials are valid)
  float slack[4];             // per-warp sum of |w_j| ||q_j||_1
};

// A [4 atoms][128 x 128 B] (q+ dims 0-63, 64-127, q- dims 0-63, 64-127),
// B [KS][4 atoms][64 x 128 B] (32 hi rows, then 32 lo rows): about 97 KB, so
// two CTAs share an SM and one's loads overlap the other's epilogue.
constexpr size_t dosa_smem_bytes() {
  return 1024 + 65536 + (size_t)kDosaKS * 32768 + sizeof(DosaSmemTail);
}

// CTA: 128 (row, head) pairs = 128 / H query rows of one sequence (TMEM lane =
// pair); the B tiles cover the blocks up to the CTA's last legal key.
__global__ void __launch_bounds__(kDosaThreads, 2)
    dosa_bound_kernel(const __grid_constant__ CUtensorMap qmap,
                      const __grid_constant__ CUtensorMap emap, const DosaArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* As = smem;
  uint8_t* Bs = As + 65536;
  DosaSmemTail* T = reinterpret_cast<DosaSmemTail*>(Bs + kDosaKS * 32768);

  const int R = 128 / a.H;                       // query rows per CTA
  const int tiles_b = (a.n_q + R - 1) / R;
  const int b = blockIdx.x / tiles_b;
  const int t0 = (blockIdx.x % tiles_b) * R;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pos0 = a.q_pos0 ? a.q_pos0[b] : a.n_tok - a.n_q;
  const int klen = a.k_len ? a.k_len[b] : a.n_tok;
  auto nblk_of = [&](int t) {                    // blocks holding row t's legal keys
    const int nleg = max(0, min(pos0 + t + 1, klen));
    return min((nleg + (1 << a.shift) - 1) >> a.shift, a.nblk);
  };
  const int nb_cta = nblk_of(min(t0 + R, a.n_q) - 1);
  const int nt = (nb_cta + kDosaBT - 1) / kDosaBT;

  if (threadIdx.x == 0) {
    mbar_init(&T->q_full, 1);
    mbar_init(&T->a_ready, 4);
    mbar_init(&T->drain, 1);
    for (int i = 0; i < kDosaKS; ++i) {
      mbar_init(&T->e_full[i], 1);
      mbar_init(&T->e_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&T->d_full[i], 1);
      mbar_init(&T->d_empty[i], 4);
    }
    T->abort = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(&T->tmem_base, 128);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    prefetch_tmap(&qmap);
    prefetch_tmap(&emap);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = T->tmem_base;
  volatile int* abort = &T->abort;

  if (warp == 4) {
    // ------------------------------------------------------------ producer --
    if (lane == 0) {
      const int prow = (b * a.n_q + t0) * a.H;
      mbar_arrive_expect_tx(&T->q_full, 32768);
      tma_load_2d(As, &qmap, &T->q_full, 0, prow);
      tma_load_2d(As + 16384, &qmap, &T->q_full, 64, prow);
      int issued = 0;
      for (int i = 0; i < nt; ++i) {
        const int slot = i % kDosaKS;
        if (!mbar_wait(&T->e_empty[slot], ((i / kDosaKS) & 1) ^ 1, abort, a.status, 150)) break;
        mbar_arrive_expect_tx(&T->e_full[slot], 32768);
        uint8_t* dst = Bs + slot * 32768;
#pragma unroll
        for (int at = 0; at < 4; ++at) {
          tma_load_3d(dst + at * 8192, &emap, &T->e_full[slot], at * 64, i * kDosaBT, b * 2);
          tma_load_3d(dst + at * 8192 + 4096, &emap, &T->e_full[slot], at * 64, i * kDosaBT,
                      b * 2 + 1);
        }
        ++issued;
      }
      if (*abort) {
        mbar_wait_drain(&T->q_full, 0);
        for (int i = issued > kDosaKS ? issued - kDosaKS : 0; i < issued; ++i)
          mbar_wait_drain(&T->e_full[i % kDosaKS], (i / kDosaKS) & 1);
      }
    }
  } else if (warp == 5) {
    // ----------------------------------------------------------------- MMA --
    if (lane == 0) {
      const uint32_t idesc = make_idesc<MmaKind::BF16>(2 * kDosaBT);
      bool ok = mbar_wait(&T->a_ready, 0, abort, a.status, 151);
      for (int i = 0; i < nt && ok; ++i) {
        const int slot = i % kDosaKS, buf = i & 1;
        if (!mbar_wait(&T->e_full[slot], (i / kDosaKS) & 1, abort, a.status, 152) ||
            !mbar_wait(&T->d_empty[buf], ((i >> 1) & 1) ^ 1, abort, a.status, 153)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t ab = smem_u32(As), bb = smem_u32(Bs + slot * 32768);
#pragma unroll
        for (int kk = 0; kk < 16; ++kk)
          tc_mma<MmaKind::BF16>(tmem + buf * (2 * kDosaBT),
                                make_sdesc(ab + (kk >> 2) * 16384 + (kk & 3) * 32),
                                make_sdesc(bb + (kk >> 2) * 8192 + (kk & 3) * 32), idesc, kk != 0);
        tc_commit(&T->e_empty[slot]);
        tc_commit(&T->d_full[buf]);
      }
      if (!ok) {
        tc_commit(&T->drain);
        mbar_wait_drain(&T->drain, 0);
      }
    }
  } else {
    // ----------------------------------------------------------- epilogue --
    const int p = threadIdx.x;                   // (row, head) pair = TMEM lane
    const int r = p / a.H, j = p % a.H;
    const int t = t0 + r;
    const bool active = t < a.n_q;
    const int64_t grow = (int64_t)b * a.n_q + t;
    const int wpr = a.H / 32;                    // warps per query row
    const bool leader = (warp % wpr) == 0;
    const float wj = active ? a.w[grow * a.H + j] : 0.f;
    bool ok = mbar_wait(&T->q_full, 0, abort, a.status, 154);
    ok = __all_sync(0xffffffffu, ok);
    // q+ over the loaded dims, q- into atoms 2 and 3 (same rows and chunk
    // positions, so the same swizzle), and ||q_j||_1
    float l1 = 0.f;
    if (ok) {
#pragma unroll
      for (int at = 0; at < 2; ++at) {
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
          const int ch = c8 ^ (p & 7);           // spread the warp over the banks
          uint4* src = reinterpret_cast<uint4*>(As + at * 16384 + p * 128 + ch * 16);
          uint4* neg = reinterpret_cast<uint4*>(As + (at + 2) * 16384 + p * 128 + ch * 16);
          uint4 v = *src;
          uint32_t* u = reinterpret_cast<uint32_t*>(&v);
          uint4 pv, nv;
          uint32_t* up = reinterpret_cast<uint32_t*>(&pv);
          uint32_t* un = reinterpret_cast<uint32_t*>(&nv);
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            const uint32_t m = ((u[x] >> 15) & 0x00010001u) * 0xFFFFu;   // sign of each half
            up[x] = u[x] & ~m;
            un[x] = u[x] & m;
            l1 += fabsf(__uint_as_float(u[x] << 16)) + fabsf(__uint_as_float(u[x] & 0xFFFF0000u));
          }
          *src = pv;
          *neg = nv;
        }
      }
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&T->a_ready);
    // slack of each row: 2^-12 sum_j |w_j| ||q_j||_1 (times mx_b per block)
    float sl = fabsf(wj) * l1;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) sl += __shfl_xor_sync(0xffffffffu, sl, o);
    if (lane == 0) T->slack[warp] = sl;
    named_bar_sync(1, 128);
    float srow = 0.f;
    for (int x = 0; x < wpr; ++x) srow += T->slack[warp - warp % wpr + x];
    srow *= 2.44140625e-04f;
    const int nb_t = active ? nblk_of(t) : 0;
    float* ubr = a.ub + grow * a.nblk;
    const float* mxb = a.mx + (int64_t)b * a.nblk;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    // every epilogue warp runs all nt rounds (the named barrier below needs all
    // four); a round whose wait failed does no work and marks its partials bad
    for (int i = 0; i < nt; ++i) {
      const int buf = i & 1;
      if (ok) ok = mbar_wait(&T->d_full[buf], (i >> 1) & 1, abort, a.status, 155);
      ok = __all_sync(0xffffffffu, ok);
      if (lane == 0) T->okw[buf][warp] = ok ? 1 : 0;
      if (!ok) {
        named_bar_sync(1, 128);
        continue;
      }
      tc_fence_after();
      uint32_t hv[32], lv[32];
      tmem_ld32(tmem + lane_off + buf * (2 * kDosaBT), hv);
      tmem_ld32(tmem + lane_off + buf * (2 * kDosaBT) + kDosaBT, lv);
      tmem_ld_wait(hv);
      tmem_ld_wait(lv);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&T->d_empty[buf]);
      // sum over the warp's 32 heads, all 32 blocks at once: each round keeps
      // one half of the values and adds the partner lane's copy of it; lane l
      // ends with block l
      auto head_sum = [&](float (&v)[32]) {
#pragma unroll
        for (int bit = 16; bit >= 1; bit >>= 1) {
          const bool up = (lane & bit) != 0;
#pragma unroll
          for (int x = 0; x < bit; ++x) {
            const float keep = up ? v[x + bit] : v[x];
            const float send = up ? v[x] : v[x + bit];
            v[x] = keep + __shfl_xor_sync(0xffffffffu, send, bit);
          }
        }
        return v[0];
      };
      float v[32];
#pragma unroll
      for (int x = 0; x < 32; ++x)
        v[x] = wj > 0.f ? wj * fmaxf(__uint_as_float(hv[x]), 0.f)
                        : wj * fmaxf(__uint_as_float(lv[x]), 0.f);
      T->part[buf][warp][lane] = head_sum(v);
      if (a.lb) {
#pragma unroll
        for (int x = 0; x < 32; ++x)
          v[x] = wj > 0.f ? wj * fmaxf(__uint_as_float(lv[x]), 0.f)
                          : wj * fmaxf(__uint_as_float(hv[x]), 0.f);
        T->partl[buf][warp][lane] = head_sum(v);
      }
      named_bar_sync(1, 128);
      if (leader && active) {
        const int blk = i * kDosaBT + lane;
        bool all = true;
        for (int x = 0; x < wpr; ++x) all = all && T->okw[buf][warp + x] != 0;
        if (all && blk < a.nblk) {
          float s = 0.f;
          for (int x = 0; x < wpr; ++x) s += T->part[buf][warp + x][lane];
          ubr[blk] = blk < nb_t ? s + srow * mxb[blk] : -__int_as_float(0x7f800000);
          if (a.lb) {
            float sl = 0.f;
            for (int x = 0; x < wpr; ++x) sl += T->partl[buf][warp + x][lane];
            a.lb[grow * a.nblk + blk] =
                blk < nb_t ? sl - srow * mxb[blk] : -__int_as_float(0x7f800000);
          }
        }
      }
    }
    // blocks past the CTA's last legal key
    if (ok && leader && active)
      for (int blk = nt * kDosaBT + lane; blk < a.nblk; blk += 32) {
        ubr[blk] = -__int_as_float(0x7f800000);
        if (a.lb) a.lb[grow * a.nblk + blk] = -__int_as_float(0x7f800000);
      }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// ------------------------------------------------------------- seed set --
// One warp per query row: the blocks of largest lower bound (ties to the lower
// block), taken until they hold `keep` of the row's legal keys; the seed is the
// last one's lower bound (-inf when the row has fewer than keep legal keys or
// the blocks run out first).  The row's keep best scores are all at least the
// seed.
// It also counts the row's blocks and those whose upper bound already lies
// below the seed (atomically, into counts[0] and counts[1]): the share the
// bounds are sure to prune, which decides whether the scan checks them.
__global__ void __launch_bounds__(256)
    dosa_seed_kernel(int32_t batch, int32_t n_q, int32_t n_tok, int32_t nblk, int32_t shift,
                     int32_t keep, const int32_t* __restrict__ q_pos0,
                     const int32_t* __restrict__ k_len, const float* __restrict__ lb,
                     const float* __restrict__ ub, float* __restrict__ seed,
                     unsigned long long* __restrict__ counts) {
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= (int64_t)batch * n_q) return;
  const int b = (int)(row / n_q), t = (int)(row % n_q);
  const int pos0 = q_pos0 ? q_pos0[b] : n_tok - n_q;
  const int klen = k_len ? k_len[b] : n_tok;
  const int nleg = max(0, min(pos0 + t + 1, klen));
  const int nb = min((nleg + (1 << shift) - 1) >> shift, nblk);
  const float* l = lb + row * nblk;
  const float ninf = -__int_as_float(0x7f800000);
  float out = ninf;
  if (nleg >= keep) {
    // descending (value, lower block first): the next pick is the largest
    // entry strictly after the previous one in that order
    float pv = __int_as_float(0x7f800000);
    int pa = -1, got = 0;
    for (int it = 0; it < nb && got < keep; ++it) {
      float bv = ninf;
      int ba = nb;
      for (int x = lane; x < nb; x += 32) {
        const float v = l[x];
        const bool after = v < pv || (v == pv && x > pa);
        if (after && (v > bv || (v == bv && x < ba))) {
          bv = v;
          ba = x;
        }
      }
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oa = __shfl_xor_sync(0xffffffffu, ba, o);
        if (ov > bv || (ov == bv && oa < ba)) {
          bv = ov;
          ba = oa;
        }
      }
      if (ba >= nb || bv == ninf) break;
      got += min(1 << shift, nleg - (ba << shift));
      pv = bv;
      pa = ba;
    }
    if (got >= keep) out = pv;
  }
  if (lane == 0) seed[row] = out;
  unsigned ruled = 0;
  const float* u = ub + row * nblk;
  for (int x = lane; x < nb; x += 32) ruled += u[x] < out ? 1u : 0u;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) ruled += __shfl_xor_sync(0xffffffffu, ruled, o);
  if (lane == 0 && nb > 0) {
    atomicAdd(&counts[0], (unsigned long long)nb);
    if (ruled) atomicAdd(&counts[1], (unsigned long long)ruled);
  }
}

}  // namespace dsa

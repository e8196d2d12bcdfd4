// resid.cuh — indexer LISA and ResMiSA: the shared linear term and the
// routed residual heads.
//
// "PaperTrace 2.2.2 MISA, LISA and ResMiSA", section 3.1: every head scores the
// same key, and ReLU(x) = x + ReLU(-x), so
//     I_{t,s} = g_t . k_s + sum_j w_{t,j} ReLU(-q_{t,j} . k_s),
//     g_t = sum_j w_{t,j} q_{t,j}  (the fused query).
// Indexer LISA ranks tokens by the linear term l_{t,s} = g_t . k_s alone;
// section 3.2's ResMiSA adds r residual heads chosen per query from bounds on
// -q_{t,j} . k over the blocks of the legal prefix:
//     U-_{t,b,j} = sum_c max(q_c, 0) (-kmin_{b,c}) + max(-q_c, 0) kmax_{b,c},
//     S_{t,j}    = |w_{t,j}| max_b ReLU(U-_{t,b,j}),
// keeps the r heads of largest S (ties to the lower head) and scores
//     I^_{t,s} = l_{t,s} + sum_{j in A_t} w_{t,j} ReLU(-q_{t,j} . k_s).
//
// Both reuse the indexer scan: each query row is rewritten as a small set of
// "pseudo-heads" whose weighted ReLU sum is exactly the method's score.  The
// linear term needs no ReLU: with g split into two bf16 parts g = g_hi + g_lo
// (about 16 significant bits), ReLU(x) - ReLU(-x) = x gives
//     l = [ReLU(g_hi.k) - ReLU(-g_hi.k)] + [ReLU(g_lo.k) - ReLU(-g_lo.k)]
// as four pseudo-heads (queries g_hi, -g_hi, g_lo, -g_lo; weights 1, -1, 1, -1),
// each an fp32 dot product on the tensor core; a residual head is the pseudo-head
// (-q_j, w_j).  Unused pseudo-heads have zero query and zero weight.
#pragma once
#include "common.cuh"

namespace dsa {

// --------------------------------------------------------- pseudo-heads --
struct PseudoArgs {
  int64_t rows;            // batch * n_q query rows
  int32_t H;               // indexer heads
  int32_t HP;              // pseudo-heads per row (power of two, >= 4 + r)
  int32_t r;               // residual heads per row (0: LISA)
  const uint16_t* q;       // [rows, H, 128] bf16
  const float* w;          // [rows, H]
  const int32_t* heads;    // [rows, r] residual heads (ascending) or null
  uint16_t* qp;            // [rows, HP, 128] bf16 pseudo-head queries
  float* wp;               // [rows, HP] pseudo-head weights
};

__device__ __forceinline__ uint16_t f32_to_bf16_rn(float x) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

// One warp per query row; lane l owns dimensions 4l .. 4l + 3.  The fused query
// is accumulated in fp32 over the heads in ascending order (fma), then split:
// hi = bf16(g), lo = bf16(g - hi), the subtraction exact in fp32.
__global__ void __launch_bounds__(256) pseudo_heads_kernel(const PseudoArgs a) {
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= a.rows) return;
  const uint16_t* qr = a.q + row * a.H * 128;
  const float* wr = a.w + row * a.H;
  float g[4] = {0.f, 0.f, 0.f, 0.f};
  for (int j = 0; j < a.H; ++j) {
    const float wj = wr[j];
    const uint2 v = *reinterpret_cast<const uint2*>(qr + j * 128 + lane * 4);
    g[0] = fmaf(wj, __uint_as_float(v.x << 16), g[0]);
    g[1] = fmaf(wj, __uint_as_float(v.x & 0xFFFF0000u), g[1]);
    g[2] = fmaf(wj, __uint_as_float(v.y << 16), g[2]);
    g[3] = fmaf(wj, __uint_as_float(v.y & 0xFFFF0000u), g[3]);
  }
  uint16_t hi[4], lo[4], nhi[4], nlo[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    hi[c] = f32_to_bf16_rn(g[c]);
    const float rest = g[c] - __uint_as_float((uint32_t)hi[c] << 16);
    lo[c] = f32_to_bf16_rn(rest);
    nhi[c] = hi[c] ^ 0x8000u;   // exact negations
    nlo[c] = lo[c] ^ 0x8000u;
  }
  auto put = [&](int p, const uint16_t (&v)[4]) {
    uint2 o;
    o.x = (uint32_t)v[0] | ((uint32_t)v[1] << 16);
    o.y = (uint32_t)v[2] | ((uint32_t)v[3] << 16);
    *reinterpret_cast<uint2*>(a.qp + (row * a.HP + p) * 128 + lane * 4) = o;
  };
  put(0, hi);
  put(1, nhi);
  put(2, lo);
  put(3, nlo);
  float* wpr = a.wp + row * a.HP;
  if (lane == 0) {
    wpr[0] = 1.f;
    wpr[1] = -1.f;
    wpr[2] = 1.f;
    wpr[3] = -1.f;
  }
  for (int p = 4; p < a.HP; ++p) {
    const int x = p - 4;
    uint2 o = make_uint2(0u, 0u);
    float wv = 0.f;
    if (x < a.r) {
      const int j = a.heads[row * a.r + x];
      const uint2 v = *reinterpret_cast<const uint2*>(qr + j * 128 + lane * 4);
      o.x = v.x ^ 0x80008000u;   // -q_j, exact
      o.y = v.y ^ 0x80008000u;
      wv = wr[j];
    }
    *reinterpret_cast<uint2*>(a.qp + (row * a.HP + p) * 128 + lane * 4) = o;
    if (lane == 0) wpr[p] = wv;
  }
}

// ------------------------------------------------------- block extrema --
// grid (blocks per sequence, batch), 128 threads: thread c owns dimension c.
// ext_full [batch, nblk_full, 256]: per full block (-kmin | kmax) over its keys;
// ext_run  [batch, n_tok, 256]: at token s, (-min | max) over s's block up to s
// (the boundary block of every query whose last legal token is s).  bf16 keys:
// minima, maxima and negations are exact.
__global__ void __launch_bounds__(128)
    block_extrema_kernel(const uint16_t* __restrict__ k, int n_tok, int bs_shift,
                         uint16_t* __restrict__ ext_run, uint16_t* __restrict__ ext_full,
                         int nblk_full) {
  const int blk = blockIdx.x, b = blockIdx.y, c = threadIdx.x;
  const int bs = 1 << bs_shift;
  const int s0 = blk << bs_shift;
  const int s1 = min(s0 + bs, n_tok);
  float mn = __int_as_float(0x7f800000), mx = -__int_as_float(0x7f800000);
  for (int sb = s0; sb < s1; sb += 8) {
    float x[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int s = min(sb + e, s1 - 1);
      x[e] = __uint_as_float((uint32_t)k[((int64_t)b * n_tok + s) * 128 + c] << 16);
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int s = sb + e;
      if (s >= s1) break;
      mn = fminf(mn, x[e]);
      mx = fmaxf(mx, x[e]);
      const int64_t off = ((int64_t)b * n_tok + s) * 256;
      const uint16_t nmn = (uint16_t)(__float_as_uint(mn) >> 16) ^ 0x8000u;
      const uint16_t pmx = (uint16_t)(__float_as_uint(mx) >> 16);
      ext_run[off + c] = nmn;
      ext_run[off + 128 + c] = pmx;
      if (s == s0 + bs - 1 && blk < nblk_full) {
        const int64_t foff = ((int64_t)b * nblk_full + blk) * 256;
        ext_full[foff + c] = nmn;
        ext_full[foff + 128 + c] = pmx;
      }
    }
  }
}

// ------------------------------------------------------ residual router --
struct ResRouterArgs {
  int32_t batch, n_q, n_tok, H, r;
  int32_t bs_shift;          // router block = 2^bs_shift tokens
  int32_t nblk_full;         // full blocks per sequence in ext_full
  const int32_t* q_pos0;     // [batch] or null: n_tok - n_q
  const int32_t* k_len;      // [batch] or null: n_tok
  const uint16_t* q;         // [batch, n_q, H, 128] bf16
  const float* w;            // [batch, n_q, H]
  const uint16_t* ext_full;  // [batch, nblk_full, 256]
  const uint16_t* ext_run;   // [batch, n_tok, 256]
  int32_t* heads;            // [batch * n_q, r] ascending
  float* S;                  // [batch * n_q, H] or null
};

constexpr int kResThreads = 256;     // one thread per (query row, head): 256 / H rows per CTA
constexpr int kResBlkTile = 8;       // full-block extrema staged per round

// CTA: 256 / H query rows of one sequence x H heads.  Each thread keeps its
// query head in registers; a block's bound is sum_c |q_c| * (q_c > 0 ? -kmin_c :
// kmax_c), accumulated in fp32 over c in ascending order.  Full-block extrema
// are staged in shared memory for all the CTA's rows, each row's boundary block
// (the extrema of its legal tokens in the last, partial block) likewise.
__global__ void __launch_bounds__(kResThreads) residual_router_kernel(const ResRouterArgs a) {
  __shared__ __align__(16) float ext[kResBlkTile][256];
  __shared__ __align__(16) float ebnd[32][256];     // per row (<= 32 rows): boundary extrema
  __shared__ float Ssm[kResThreads];
  __shared__ int sel_sm[kResThreads];
  const int rpc = kResThreads / a.H;                  // rows per CTA
  const int tiles = (a.n_q + rpc - 1) / rpc;
  const int b = blockIdx.x / tiles;
  const int t0 = (blockIdx.x % tiles) * rpc;
  const int ri = threadIdx.x / a.H, j = threadIdx.x % a.H;
  const int t = t0 + ri;
  const bool active = t < a.n_q;
  const int pos0 = a.q_pos0 ? a.q_pos0[b] : a.n_tok - a.n_q;
  const int klen = a.k_len ? a.k_len[b] : a.n_tok;
  const int nleg = active ? max(0, min(pos0 + t + 1, klen)) : 0;
  const int nfull = min(nleg >> a.bs_shift, a.nblk_full);
  const bool has_bnd = nleg > (nfull << a.bs_shift);
  // the CTA's rows share full blocks up to the largest count among them (the last row's)
  const int tl = min(t0 + rpc, a.n_q) - 1;
  const int nfull_cta = min(max(0, min(pos0 + tl + 1, klen)) >> a.bs_shift, a.nblk_full);
  const int64_t row = (int64_t)b * a.n_q + t;
  // boundary extrema of every row of the CTA
  for (int i = threadIdx.x; i < rpc * 256; i += kResThreads) {
    const int rr = i >> 8, c = i & 255;
    const int tt = t0 + rr;
    float v = 0.f;
    if (tt < a.n_q) {
      const int nl = max(0, min(pos0 + tt + 1, klen));
      if (nl > 0) v = __uint_as_float((uint32_t)a.ext_run[((int64_t)b * a.n_tok + nl - 1) * 256 + c] << 16);
    }
    ebnd[rr][c] = v;
  }
  float q[128];
  {
    const uint16_t* qr = a.q + ((active ? row : (int64_t)b * a.n_q) * a.H + j) * 128;
#pragma unroll
    for (int c = 0; c < 128; c += 8) {
      const uint4 v = *reinterpret_cast<const uint4*>(qr + c);
      q[c + 0] = __uint_as_float(v.x << 16);
      q[c + 1] = __uint_as_float(v.x & 0xFFFF0000u);
      q[c + 2] = __uint_as_float(v.y << 16);
      q[c + 3] = __uint_as_float(v.y & 0xFFFF0000u);
      q[c + 4] = __uint_as_float(v.z << 16);
      q[c + 5] = __uint_as_float(v.z & 0xFFFF0000u);
      q[c + 6] = __uint_as_float(v.w << 16);
      q[c + 7] = __uint_as_float(v.w & 0xFFFF0000u);
    }
  }
  // U- of one block from its staged extrema e = (-kmin | kmax)
  auto bound = [&](const float* e) {
    float u = 0.f;
#pragma unroll
    for (int c = 0; c < 128; ++c) u = fmaf(fabsf(q[c]), q[c] > 0.f ? e[c] : e[128 + c], u);
    return u;
  };
  float best = 0.f;   // max_b ReLU(U-): starts at 0
  for (int b0 = 0; b0 < nfull_cta; b0 += kResBlkTile) {
    const int nb = min(kResBlkTile, nfull_cta - b0);
    __syncthreads();
    for (int i = threadIdx.x; i < nb * 256; i += kResThreads) {
      const int bb = i >> 8, c = i & 255;
      ext[bb][c] = __uint_as_float(
          (uint32_t)a.ext_full[((int64_t)b * a.nblk_full + b0 + bb) * 256 + c] << 16);
    }
    __syncthreads();
    for (int bb = 0; bb < nb && b0 + bb < nfull; ++bb) best = fmaxf(best, bound(ext[bb]));
  }
  __syncthreads();
  if (has_bnd) best = fmaxf(best, bound(ebnd[ri]));
  const float s = active ? fabsf(a.w[row * a.H + j]) * best : 0.f;
  if (active && a.S) a.S[row * a.H + j] = s;
  Ssm[threadIdx.x] = s;
  __syncthreads();
  // rank of head j among its row: heads with a larger S, or an equal S and a lower index
  const float* Sr = Ssm + ri * a.H;
  int rank = 0;
  for (int i = 0; i < a.H; ++i) {
    const float o = Sr[i];
    rank += (o > s || (o == s && i < j)) ? 1 : 0;
  }
  sel_sm[threadIdx.x] = rank < a.r ? 1 : 0;
  __syncthreads();
  if (!active || rank >= a.r) return;
  int below = 0;   // selected heads below j: the ascending position of j
  for (int i = 0; i < j; ++i) below += sel_sm[ri * a.H + i];
  a.heads[row * a.r + below] = j;
}

}  // namespace dsa

// bwd.cuh — indexer backward with score recompute over the selected positions.
//
// "PaperTrace 2.2.2 MISA, LISA and ResMiSA", section 2.3 "why training
// gradients need recomputation": the forward keeps only the selected positions
// S_t; the backward recomputes z_{t,s,j} = q_{t,j} . k_s with the mask
// m = 1[z > 0] (ReLU's derivative is 0 at 0) and, for an upstream gradient
// g_{t,s} on I_{t,s}, forms
//     dq_{t,j} = sum_{s in S_t} g_{t,s} w_{t,j} m_{t,s,j} k_s
//     dk_s     = sum_t sum_j    g_{t,s} w_{t,j} m_{t,s,j} q_{t,j}
//     dw_{t,j} = sum_{s in S_t} g_{t,s} ReLU(z_{t,s,j}).
//
// One CTA per query row t (64 heads, d = 128); its selected rows stream in
// tiles of 128 positions gathered four rows per TMA copy.  Per tile, on tcgen05:
//   Z   = K . Q_t^T    M = 128 positions, N = 64 heads, K = 128   (recompute)
//   dQ += G'^T . K     M = 128 (64 head rows + 64 zero rows), N = 128 dims,
//                      K = 128 positions; K read as an MN-major operand
//   dK  = G' . Q_t     M = 128 positions, N = 128 dims, K = 64 heads; Q_t read
//                      as an MN-major operand
// with G'_{s,j} = g_s w_j 1[z > 0] (bf16) written by the epilogue both ways
// (position-major for dK, head-major for dQ).  dw is reduced in fp32 from Z
// directly.  Each tile's dK rows are added to the key gradients with vector
// reductions (several rows select the same key).  Warps 0-3: epilogue (thread =
// position of the tile); warp 4: TMA producer; warp 5: MMA issuer.
#pragma once
#include "common.cuh"

namespace dsa {

constexpr int kBwdH = 64;
constexpr int kBwdTile = 128;          // positions per tile
constexpr int kBwdKS = 3;              // key-tile pipeline depth
constexpr int kBwdThreads = 192;

struct BwdArgs {
  int32_t rows;          // batch * n_q query rows
  int32_t n_q, n_k;
  int32_t topk;
  const int32_t* sel;    // [rows, topk] selected positions (-1: empty)
  const float* grad;     // [rows, topk] upstream gradient on I at those positions
  const float* w;        // [rows, 64]
  float* dq;             // [rows, 64, 128] (written)
  float* dk;             // [batch, n_k, 128] (accumulated)
  float* dw;             // [rows, 64] (written)
  int32_t* status;
};

struct BwdSmemTail {
  uint64_t q_full, z_full[2], z_empty[2], g_full, g_free, dk_full, dk_empty, drain;
  uint64_t k_full[kBwdKS], k_empty[kBwdKS];
  uint32_t tmem_base;
  int32_t abort;
  float dw_acc[kBwdH];
  float wrow[kBwdH];
};

// Shared memory: Q tile [2 atoms][64 rows x 128 B], key tiles [KS][2 atoms][128 x 128 B],
// G' [128 positions x 128 B], G'^T [2 atoms][128 rows x 128 B] (rows 64-127 zero).
constexpr size_t bwd_smem_bytes() {
  return 1024 + 16384 + (size_t)kBwdKS * 32768 + 16384 + 32768 + sizeof(BwdSmemTail);
}

__device__ __forceinline__ uint64_t make_sdesc_mn_b(uint32_t smem_addr, uint32_t lbo) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr >> 4) & 0x3FFF);
  d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

__global__ void __launch_bounds__(kBwdThreads, 1)
    indexer_backward_kernel(const __grid_constant__ CUtensorMap qmap,
                            const __grid_constant__ CUtensorMap kmap, const BwdArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* Qs = smem;                              // [2][64 x 128 B]
  uint8_t* Ks = Qs + 16384;                        // [KS][2][128 x 128 B]
  uint8_t* Gs = Ks + kBwdKS * 32768;               // [128 x 128 B]   position-major
  uint8_t* GTs = Gs + 16384;                       // [2][128 x 128 B] head-major
  BwdSmemTail* T = reinterpret_cast<BwdSmemTail*>(GTs + 32768);

  const int row = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nt = (a.topk + kBwdTile - 1) / kBwdTile;
  const int32_t* sel_r = a.sel + (int64_t)row * a.topk;
  const float* g_r = a.grad + (int64_t)row * a.topk;
  const int krow0 = (row / a.n_q) * a.n_k;

  if (threadIdx.x == 0) {
    mbar_init(&T->q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&T->z_full[i], 1);
      mbar_init(&T->z_empty[i], 4);
    }
    mbar_init(&T->g_full, 4);
    mbar_init(&T->g_free, 1);
    mbar_init(&T->dk_full, 1);
    mbar_init(&T->dk_empty, 4);
    mbar_init(&T->drain, 1);
    for (int i = 0; i < kBwdKS; ++i) {
      mbar_init(&T->k_full[i], 1);
      mbar_init(&T->k_empty[i], 1);
    }
    T->abort = 0;
    fence_barrier_init();
  }
  // zero the head-major G'^T (its rows 64-127 stay zero) and the dw sums
  for (int i = threadIdx.x; i < 32768 / 16; i += kBwdThreads)
    reinterpret_cast<uint4*>(GTs)[i] = make_uint4(0u, 0u, 0u, 0u);
  if (threadIdx.x < kBwdH) {
    T->dw_acc[threadIdx.x] = 0.f;
    T->wrow[threadIdx.x] = a.w[(int64_t)row * kBwdH + threadIdx.x];
  }
  fence_proxy_async_smem();
  if (warp == 5) {
    tmem_alloc(&T->tmem_base, 512);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    prefetch_tmap(&qmap);
    prefetch_tmap(&kmap);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = T->tmem_base;
  // TMEM columns: Z [0, 128) (two buffers of 64), dQ [128, 256), dK [256, 384)
  const uint32_t tm_dq = tmem + 128, tm_dk = tmem + 256;
  volatile int* abort = &T->abort;

  if (warp == 4) {
    // ------------------------------------------------------------ producer --
    bool ok = true;
    if (lane == 0) {
      mbar_arrive_expect_tx(&T->q_full, 16384);
      for (int at = 0; at < 2; ++at)
        tma_load_2d(Qs + at * 8192, &qmap, &T->q_full, at * 64, row * kBwdH);
    }
    uint32_t kc = 0;
    for (int i = 0; i < nt && ok; ++i) {
      // lane l gathers positions 4l .. 4l + 3 of the tile
      int r[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int e = i * kBwdTile + lane * 4 + j;
        int s = e < a.topk ? sel_r[e] : -1;
        if (s >= a.n_k) {
          set_status(a.status, DSA_ERR_INTERNAL, 140);
          s = -1;
        }
        r[j] = krow0 + (s > 0 ? s : 0);
      }
      const int slot = kc % kBwdKS;
      if (lane == 0) {
        ok = mbar_wait(&T->k_empty[slot], ((kc / kBwdKS) & 1) ^ 1, abort, a.status, 41);
        if (ok) mbar_arrive_expect_tx(&T->k_full[slot], 32768);
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      for (int at = 0; at < 2; ++at)
        tma_gather4(Ks + slot * 32768 + at * 16384 + lane * 512, &kmap, &T->k_full[slot],
                    at * 64, r[0], r[1], r[2], r[3]);
      ++kc;
    }
    if (lane == 0 && *abort) {
      mbar_wait_drain(&T->q_full, 0);
      for (uint32_t i = kc > (uint32_t)kBwdKS ? kc - kBwdKS : 0; i < kc; ++i)
        mbar_wait_drain(&T->k_full[i % kBwdKS], (i / kBwdKS) & 1);
    }
  } else if (warp == 5) {
    // ----------------------------------------------------------------- MMA --
    if (lane == 0) {
      const uint32_t idesc_z = make_idesc<MmaKind::BF16>(kBwdH);
      const uint32_t idesc_dq = make_idesc<MmaKind::BF16>(128) | (1u << 16);   // B MN-major
      const uint32_t idesc_dk = make_idesc<MmaKind::BF16>(128) | (1u << 16);   // B MN-major
      bool ok = mbar_wait(&T->q_full, 0, abort, a.status, 42);
      // Z of tile i into buffer i & 1
      auto issue_z = [&](int i) -> bool {
        const int b = i & 1, slot = i % kBwdKS;
        if (!mbar_wait(&T->z_empty[b], ((i >> 1) & 1) ^ 1, abort, a.status, 43)) return false;
        if (!mbar_wait(&T->k_full[slot], (i / kBwdKS) & 1, abort, a.status, 44)) return false;
        tc_fence_after();
        const uint32_t kb = smem_u32(Ks + slot * 32768);
#pragma unroll
        for (int at = 0; at < 2; ++at)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            tc_mma<MmaKind::BF16>(tmem + b * kBwdH, make_sdesc(kb + at * 16384 + kk * 32),
                                  make_sdesc(smem_u32(Qs) + at * 8192 + kk * 32), idesc_z,
                                  (at | kk) != 0);
        tc_commit(&T->z_full[b]);
        return true;
      };
      if (ok && nt > 0) ok = issue_z(0);
      for (int i = 0; i < nt && ok; ++i) {
        if (i + 1 < nt && !issue_z(i + 1)) {
          ok = false;
          break;
        }
        // G' of tile i written, the previous dK tile read out
        if (!mbar_wait(&T->g_full, i & 1, abort, a.status, 45) ||
            !mbar_wait(&T->dk_empty, (i & 1) ^ 1, abort, a.status, 46)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int slot = i % kBwdKS;
        const uint32_t kb = smem_u32(Ks + slot * 32768);
        // dQ (head rows) += G'^T . K: A head-major G'^T (K-major over positions),
        // B the key tile as an MN-major operand (dims contiguous, 64-dim blocks 16 KB apart)
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          tc_mma<MmaKind::BF16>(tm_dq,
                                make_sdesc(smem_u32(GTs) + (kk >> 2) * 16384 + (kk & 3) * 32),
                                make_sdesc_mn_b(kb + kk * 2048, 16384), idesc_dq, (i | kk) != 0);
        // dK = G' . Q_t: A position-major G' (K-major over heads), B the query tile as
        // an MN-major operand (dims contiguous, 64-dim blocks 8 KB apart)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          tc_mma<MmaKind::BF16>(tm_dk, make_sdesc(smem_u32(Gs) + kk * 32),
                                make_sdesc_mn_b(smem_u32(Qs) + kk * 2048, 8192), idesc_dk, kk != 0);
        tc_commit(&T->k_empty[slot]);
        tc_commit(&T->g_free);
        tc_commit(&T->dk_full);
      }
      if (!ok) {
        tc_commit(&T->drain);
        mbar_wait_drain(&T->drain, 0);
      }
    }
  } else {
    // ----------------------------------------------------------- epilogue --
    const int p = threadIdx.x;                       // position within the tile = TMEM lane
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const float* wv = T->wrow;
    bool ok = true;
    for (int i = 0; i < nt && ok; ++i) {
      const int e = i * kBwdTile + p;
      const int s = e < a.topk ? sel_r[e] : -1;
      const bool valid = s >= 0 && s < a.n_k;
      const float g = valid ? g_r[e] : 0.f;
      ok = mbar_wait(&T->z_full[i & 1], (i >> 1) & 1, abort, a.status, 47);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      uint32_t zv[2][32];
      tmem_ld32(tmem + lane_off + (i & 1) * kBwdH, zv[0]);
      tmem_ld32(tmem + lane_off + (i & 1) * kBwdH + 32, zv[1]);
      tmem_ld_wait(zv[0]);
      tmem_ld_wait(zv[1]);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&T->z_empty[i & 1]);
      // the G' buffers are free once the previous tile's dQ / dK MMAs are done
      if (i > 0) {
        ok = mbar_wait(&T->g_free, (i - 1) & 1, abort, a.status, 48);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
      }
      float dwp[kBwdH];
      uint8_t* grow = Gs + p * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint32_t w4[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          uint32_t pair = 0u;
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const int j = c * 8 + u * 2 + h2;
            const float z = __uint_as_float(zv[j >> 5][j & 31]);
            dwp[j] = g * fmaxf(z, 0.f);
            const float gp = z > 0.f ? g * wv[j] : 0.f;
            const uint16_t bits = __bfloat16_as_ushort(__float2bfloat16_rn(gp));
            pair |= (uint32_t)bits << (16 * h2);
            // head-major copy: row j, position p (atom p / 64, 16-byte chunk (p % 64) / 8)
            const int at = p >> 6, pc = (p & 63) >> 3;
            *reinterpret_cast<uint16_t*>(GTs + at * 16384 + j * 128 + ((pc ^ (j & 7)) << 4) +
                                         (p & 7) * 2) = bits;
          }
          w4[u] = pair;
        }
        *reinterpret_cast<uint4*>(grow + ((c ^ (p & 7)) << 4)) =
            make_uint4(w4[0], w4[1], w4[2], w4[3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&T->g_full);
      // dw: sum over the 128 positions per head, a reduce-scatter across the warp
      // (each round keeps one half of the values and adds the partner's copy of
      // it; lanes end with two heads each), then across the four warps in smem
      {
        int n = kBwdH;
#pragma unroll
        for (int bit = 16; bit >= 1; bit >>= 1) {
          const bool hi = (lane & bit) != 0;
          n >>= 1;
#pragma unroll
          for (int x = 0; x < kBwdH / 2; ++x) {
            if (x >= n) break;
            const float keep = hi ? dwp[x + n] : dwp[x];
            const float send = hi ? dwp[x] : dwp[x + n];
            dwp[x] = keep + __shfl_xor_sync(0xffffffffu, send, bit);
          }
        }
        int base = 0, span = kBwdH;
#pragma unroll
        for (int bit = 16; bit >= 1; bit >>= 1) {
          span >>= 1;
          if (lane & bit) base += span;
        }
        atomicAdd(&T->dw_acc[base + 0], dwp[0]);
        atomicAdd(&T->dw_acc[base + 1], dwp[1]);
      }
      // dK of this tile: add each position's row to the key gradient
      ok = mbar_wait(&T->dk_full, i & 1, abort, a.status, 49);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      float* dkrow = a.dk + ((int64_t)krow0 + (valid ? s : 0)) * 128;
      for (int c0 = 0; c0 < 128; c0 += 32) {
        uint32_t dv[32];
        tmem_ld32(tm_dk + lane_off + c0, dv);
        tmem_ld_wait(dv);
        if (valid) {
#pragma unroll
          for (int x = 0; x < 32; x += 4)
            asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dkrow + c0 + x),
                         "f"(__uint_as_float(dv[x])), "f"(__uint_as_float(dv[x + 1])),
                         "f"(__uint_as_float(dv[x + 2])), "f"(__uint_as_float(dv[x + 3]))
                         : "memory");
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&T->dk_empty);
    }
    // dQ (TMEM lanes 0-63 = heads, columns = dims) and dw of the row
    if (ok && nt > 0) {
      ok = mbar_wait(&T->g_free, (nt - 1) & 1, abort, a.status, 50);
      ok = __all_sync(0xffffffffu, ok);
    }
    named_bar_sync(1, 128);
    if (ok) {
      tc_fence_after();
      if (warp < 2) {
        float* dqr = a.dq + ((int64_t)row * kBwdH + p) * 128;
        for (int c0 = 0; c0 < 128; c0 += 32) {
          uint32_t dv[32];
          if (nt > 0) {
            tmem_ld32(tm_dq + lane_off + c0, dv);
            tmem_ld_wait(dv);
          } else {
#pragma unroll
            for (int x = 0; x < 32; ++x) dv[x] = 0u;
          }
#pragma unroll
          for (int x = 0; x < 32; x += 4)
            *reinterpret_cast<float4*>(dqr + c0 + x) =
                make_float4(__uint_as_float(dv[x]), __uint_as_float(dv[x + 1]),
                            __uint_as_float(dv[x + 2]), __uint_as_float(dv[x + 3]));
        }
      }
      if (p < kBwdH) a.dw[(int64_t)row * kBwdH + p] = T->dw_acc[p];
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace dsa

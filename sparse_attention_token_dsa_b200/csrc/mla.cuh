// mla.cuh — Sparse MLA attention over a fixed set of selected positions.
//
// "PaperTrace 2.2.2 MISA, LISA and ResMiSA", section 2.2: the indexer's top-k
// positions feed Sparse MLA, which reads the latent KV at those (scattered)
// positions; section 2.3, acceptance step two: with the candidate set fixed,
// the attention must reproduce a naive gather attention's logits, row
// maximum, softmax denominator and output.  For token t with query heads q_h
// (the absorbed MLA query: latent part and rope part, 576 dimensions) and the
// cached rows kv_s (latent 512 + rope 64) of its selected positions s:
//     x_s = scale q_h . kv_s,   o_h = sum_s softmax(x)_s kv_s[0:512],
//     lse_h = log sum_s exp(x_s).
//
// One CTA per (token, half of the 512 value dimensions); 128 query-head rows
// (TMEM lane = head; fewer heads are zero rows).  The query tile stays in
// shared memory (9 chunks of 64 dimensions); the selected rows stream in tiles
// of 64 positions, gathered four rows per TMA copy:
//   S  = Q . K^T   tcgen05, M = 128 heads, N = 64 positions, K = 576, two TMEM
//                  buffers so S of the next tile runs while this one is reduced
//   P  = exp2(S * scale * log2 e - m)   one thread per head row, bf16 into smem
//   O += P . V     tcgen05, N = 256 value dimensions, V read as an MN-major
//                  operand straight from the gathered rows (no transpose)
// The running maximum m is raised lazily (only when a tile's maximum exceeds
// it by more than 8 in log2 units, so P <= 256); O and the denominator are then
// rescaled.  The result o = O / l is exact up to rounding for any m.
// Warps 0-3: softmax and output; warp 4: TMA producer; warp 5: MMA issuer.
#pragma once
#include "common.cuh"

namespace dsa {

constexpr int kMlaDqk = 576;            // 512 latent + 64 rope dimensions
constexpr int kMlaDv = 512;             // value = the latent part
constexpr int kMlaQChunks = kMlaDqk / 64;
constexpr int kMlaBK = 64;              // positions per tile
constexpr int kMlaKS = 3;               // key-chunk pipeline depth
constexpr int kMlaThreads = 192;
constexpr float kMlaLazy = 8.f;         // log2 headroom before the maximum is raised

struct MlaArgs {
  int32_t T;             // query tokens
  int32_t tps;           // tokens per sequence: token t reads sequence t / tps
  int32_t n_k;           // cached rows per sequence
  int32_t heads;         // query heads (<= 128)
  int32_t topk;          // entries per token in idx
  float scale_log2;      // softmax scale * log2(e)
  const int32_t* idx;    // [T, topk] selected positions (-1: empty)
  uint16_t* out;         // [T, heads, 512] bf16
  float* lse;            // [T, heads] natural-log sum of exponentials, or null
  int32_t* status;       // workspace status word
};

struct MlaSmemTail {
  uint64_t q_full, v_full, p_full, pv_done, drain;
  uint64_t k_full[kMlaKS], k_empty[kMlaKS];
  uint64_t s_full[2], s_empty[2];
  uint32_t tmem_base;
  int32_t abort;
};

constexpr size_t mla_smem_bytes() {
  return 1024 + (size_t)kMlaQChunks * 16384 + (size_t)kMlaKS * 8192 + 4 * 8192 + 16384 +
         sizeof(MlaSmemTail);
}


// Shared-memory descriptor of an MN-major operand in 128-byte swizzled rows:
// each 128-byte row holds 64 consecutive MN elements of one K index, 8 rows form
// a 1024-byte atom (SBO = 1024 between K groups of 8), and MN blocks of 64
// elements lie `lbo` bytes apart.
__device__ __forceinline__ uint64_t make_sdesc_mn(uint32_t smem_addr, uint32_t lbo) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr >> 4) & 0x3FFF);
  d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__global__ void __launch_bounds__(kMlaThreads, 1)
    sparse_mla_kernel(const __grid_constant__ CUtensorMap qmap,
                      const __grid_constant__ CUtensorMap kvmap, const MlaArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* Qs = smem;                                   // [9][128 rows x 128 B]
  uint8_t* Ks = Qs + kMlaQChunks * 16384;               // [KS][64 rows x 128 B]
  uint8_t* Vs = Ks + kMlaKS * 8192;                     // [4][64 rows x 128 B]
  uint8_t* Ps = Vs + 4 * 8192;                          // [128 rows x 128 B]
  MlaSmemTail* T = reinterpret_cast<MlaSmemTail*>(Ps + 16384);

  const int t = blockIdx.x >> 1, hv = blockIdx.x & 1;   // token, value half
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nt = (a.topk + kMlaBK - 1) / kMlaBK;
  const int32_t* idx_t = a.idx + (int64_t)t * a.topk;
  const int krow0 = (t / a.tps) * a.n_k;

  if (threadIdx.x == 0) {
    mbar_init(&T->q_full, 1);
    mbar_init(&T->v_full, 1);
    mbar_init(&T->p_full, 4);
    mbar_init(&T->pv_done, 1);
    mbar_init(&T->drain, 1);
    for (int i = 0; i < kMlaKS; ++i) {
      mbar_init(&T->k_full[i], 1);
      mbar_init(&T->k_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&T->s_full[i], 1);
      mbar_init(&T->s_empty[i], 4);
    }
    T->abort = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(&T->tmem_base, 512);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    prefetch_tmap(&qmap);
    prefetch_tmap(&kvmap);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = T->tmem_base;
  volatile int* abort = &T->abort;

  if (warp == 4) {
    // ------------------------------------------------------------ producer --
    // Lane l < 16 gathers rows 4l .. 4l + 3 of each tile; lane 0 owns the barriers.
    bool ok = true;
    if (lane == 0) {
      mbar_arrive_expect_tx(&T->q_full, kMlaQChunks * 16384);
      for (int c = 0; c < kMlaQChunks; ++c)
        tma_load_3d(Qs + c * 16384, &qmap, &T->q_full, c * 64, 0, t);
    }
    uint32_t kc = 0;
    int vloads = 0;
    for (int i = 0; i < nt && ok; ++i) {
      int r[4] = {krow0, krow0, krow0, krow0};
      if (lane < 16) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int e = i * kMlaBK + lane * 4 + j;
          int s = e < a.topk ? idx_t[e] : -1;
          if (s >= a.n_k) {
            set_status(a.status, DSA_ERR_INTERNAL, 130);
            s = -1;
          }
          r[j] = krow0 + (s > 0 ? s : 0);    // empty entries read row 0 (masked later)
        }
      }
      for (int c = 0; c < kMlaQChunks; ++c) {
        const int slot = kc % kMlaKS;
        if (lane == 0) {
          ok = mbar_wait(&T->k_empty[slot], ((kc / kMlaKS) & 1) ^ 1, abort, a.status, 31);
          if (ok) mbar_arrive_expect_tx(&T->k_full[slot], 8192);
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        if (lane < 16)
          tma_gather4(Ks + slot * 8192 + lane * 512, &kvmap, &T->k_full[slot], c * 64, r[0], r[1],
                      r[2], r[3]);
        ++kc;
      }
      if (!ok) break;
      // the value rows of this tile (this CTA's 256 dimensions) once PV of the
      // previous tile has released the buffer
      if (lane == 0) {
        ok = i == 0 || mbar_wait(&T->pv_done, (i - 1) & 1, abort, a.status, 32);
        if (ok) mbar_arrive_expect_tx(&T->v_full, 4 * 8192);
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      if (lane < 16)
        for (int db = 0; db < 4; ++db)
          tma_gather4(Vs + db * 8192 + lane * 512, &kvmap, &T->v_full, hv * 256 + db * 64, r[0],
                      r[1], r[2], r[3]);
      ++vloads;
    }
    if (lane == 0 && *abort) {
      // abort path: let this CTA's own copies in flight land before exit
      mbar_wait_drain(&T->q_full, 0);
      for (uint32_t i = kc > (uint32_t)kMlaKS ? kc - kMlaKS : 0; i < kc; ++i)
        mbar_wait_drain(&T->k_full[i % kMlaKS], (i / kMlaKS) & 1);
      if (vloads > 0) mbar_wait_drain(&T->v_full, (vloads - 1) & 1);
    }
  } else if (warp == 5) {
    // ----------------------------------------------------------------- MMA --
    if (lane == 0) {
      const uint32_t idesc_s = make_idesc<MmaKind::BF16>(kMlaBK);
      const uint32_t idesc_pv = make_idesc<MmaKind::BF16>(256) | (1u << 16);  // B MN-major
      uint32_t kc = 0;
      bool ok = mbar_wait(&T->q_full, 0, abort, a.status, 33);
      auto issue_s = [&](int i) -> bool {
        const int b = i & 1;
        if (!mbar_wait(&T->s_empty[b], ((i >> 1) & 1) ^ 1, abort, a.status, 34)) return false;
        tc_fence_after();
        const uint32_t d = tmem + 256 + b * kMlaBK;
        for (int c = 0; c < kMlaQChunks; ++c) {
          const int slot = kc % kMlaKS;
          if (!mbar_wait(&T->k_full[slot], (kc / kMlaKS) & 1, abort, a.status, 35)) return false;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = make_sdesc(smem_u32(Qs + c * 16384) + kk * 32);
            const uint64_t bd = make_sdesc(smem_u32(Ks + slot * 8192) + kk * 32);
            tc_mma<MmaKind::BF16>(d, ad, bd, idesc_s, (c | kk) != 0);
          }
          tc_commit(&T->k_empty[slot]);
          ++kc;
        }
        tc_commit(&T->s_full[b]);
        return true;
      };
      if (ok && nt > 0) ok = issue_s(0);
      for (int i = 0; i < nt && ok; ++i) {
        if (i + 1 < nt && !issue_s(i + 1)) {
          ok = false;
          break;
        }
        if (!mbar_wait(&T->p_full, i & 1, abort, a.status, 36) ||
            !mbar_wait(&T->v_full, i & 1, abort, a.status, 37)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t ad = make_sdesc(smem_u32(Ps) + kk * 32);
          const uint64_t bd = make_sdesc_mn(smem_u32(Vs) + kk * 2048, 8192);
          tc_mma<MmaKind::BF16>(tmem, ad, bd, idesc_pv, (i | kk) != 0);
        }
        tc_commit(&T->pv_done);
      }
      if (!ok) {
        // abort path: wait for the MMAs already issued before TMEM is freed
        tc_commit(&T->drain);
        mbar_wait_drain(&T->drain, 0);
      }
    }
  } else {
    // ------------------------------------------------- softmax and output --
    const int h = threadIdx.x;                          // head row = TMEM lane
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    float m_run = -__int_as_float(0x7f800000);          // log2 units
    float l_run = 0.f;
    bool ok = true;
    for (int i = 0; i < nt && ok; ++i) {
      ok = mbar_wait(&T->s_full[i & 1], (i >> 1) & 1, abort, a.status, 38);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      uint32_t sv[2][32];
      tmem_ld32(tmem + lane_off + 256 + (i & 1) * kMlaBK, sv[0]);
      tmem_ld32(tmem + lane_off + 256 + (i & 1) * kMlaBK + 32, sv[1]);
      tmem_ld_wait(sv[0]);
      tmem_ld_wait(sv[1]);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&T->s_empty[i & 1]);
      // logits in log2 units; empty entries and the tail past topk are -inf
      float x[64];
      float mt = -__int_as_float(0x7f800000);
#pragma unroll
      for (int j4 = 0; j4 < 64; j4 += 4) {
        int4 e4 = make_int4(-1, -1, -1, -1);
        const int e = i * kMlaBK + j4;
        if (e + 3 < a.topk && (a.topk & 3) == 0) {     // 16-byte aligned rows only
          e4 = __ldg(reinterpret_cast<const int4*>(idx_t + e));
        } else {
          if (e + 0 < a.topk) e4.x = idx_t[e + 0];
          if (e + 1 < a.topk) e4.y = idx_t[e + 1];
          if (e + 2 < a.topk) e4.z = idx_t[e + 2];
          if (e + 3 < a.topk) e4.w = idx_t[e + 3];
        }
        const int ev[4] = {e4.x, e4.y, e4.z, e4.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int j = j4 + u;
          const float sj = __uint_as_float(sv[j >> 5][j & 31]);
          const bool valid = ev[u] >= 0 && ev[u] < a.n_k;
          x[j] = valid ? sj * a.scale_log2 : -__int_as_float(0x7f800000);
          mt = fmaxf(mt, x[j]);
        }
      }
      // P and O of the previous tile are free once its PV has completed
      if (i > 0) {
        ok = mbar_wait(&T->pv_done, (i - 1) & 1, abort, a.status, 39);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
      }
      // raise the running maximum of this row; O and l are rescaled by
      // f = exp2(m_old - m_new).  tcgen05.ld / st are warp-collective, so the
      // whole warp runs the rescale pass when any of its rows needs it (the
      // other rows multiply by exactly 1).
      float f = 1.f;
      const bool raise = mt > m_run + kMlaLazy;
      if (raise) {
        if (l_run > 0.f) {
          f = exp2f(m_run - mt);
          l_run *= f;
        }
        m_run = mt;
      }
      if (__any_sync(0xffffffffu, f != 1.f)) {
        for (int c0 = 0; c0 < 256; c0 += 32) {
          uint32_t ov[32];
          tmem_ld32(tmem + lane_off + c0, ov);
          tmem_ld_wait(ov);
#pragma unroll
          for (int j = 0; j < 32; ++j) ov[j] = __float_as_uint(__uint_as_float(ov[j]) * f);
          tmem_st32(tmem + lane_off + c0, ov);
        }
        tmem_st_wait();
      }
      // P row: exp2(x - m) in bf16, 128-byte swizzled K-major row h
      uint8_t* prow = Ps + h * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint32_t w4[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int j = c * 8 + u * 2;
          // empty entries (x = -inf) weigh 0, also while m is still -inf
          const float p0 = x[j] == -__int_as_float(0x7f800000) ? 0.f : exp2f(x[j] - m_run);
          const float p1 = x[j + 1] == -__int_as_float(0x7f800000) ? 0.f : exp2f(x[j + 1] - m_run);
          const __nv_bfloat16 b0 = __float2bfloat16_rn(p0), b1 = __float2bfloat16_rn(p1);
          l_run += __bfloat162float(b0) + __bfloat162float(b1);
          w4[u] = (uint32_t)__bfloat16_as_ushort(b0) | ((uint32_t)__bfloat16_as_ushort(b1) << 16);
        }
        *reinterpret_cast<uint4*>(prow + ((c ^ (h & 7)) << 4)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&T->p_full);
    }
    if (ok && nt > 0) {
      ok = mbar_wait(&T->pv_done, (nt - 1) & 1, abort, a.status, 40);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      tc_fence_after();
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
      uint16_t* orow = a.out + ((int64_t)t * a.heads + h) * kMlaDv + hv * 256;
      for (int c0 = 0; c0 < 256; c0 += 32) {
        uint32_t ov[32];
        if (nt > 0) {
          tmem_ld32(tmem + lane_off + c0, ov);
          tmem_ld_wait(ov);
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) ov[j] = 0u;
        }
        if (h < a.heads) {
#pragma unroll
          for (int j = 0; j < 32; j += 8) {
            uint32_t w4[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const float o0 = __uint_as_float(ov[j + 2 * u]) * inv;
              const float o1 = __uint_as_float(ov[j + 2 * u + 1]) * inv;
              w4[u] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(o0)) |
                      ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(o1)) << 16);
            }
            *reinterpret_cast<uint4*>(orow + c0 + j) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
          }
        }
      }
      if (hv == 0 && a.lse && h < a.heads)
        a.lse[(int64_t)t * a.heads + h] =
            l_run > 0.f ? (m_run + log2f(l_run)) * 0.6931471805599453f : -__int_as_float(0x7f800000);
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

// dsaidx.cu — C ABI of the B200 DSA lightning-indexer library (see
// include/dsaidx.h for the contract).  Host code here only validates
// arguments, plans the launch, carves the caller's workspace, encodes TMA
// descriptors and launches the kernels; every step of the computation runs on
// the GPU.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stddef.h>
#include <string.h>

#include <algorithm>

#include <mutex>

#include "../../include/dsaidx.h"
#include "common.cuh"
#include "bwd.cuh"
#include "dosa.cuh"
#include "finalize.cuh"
#include "mla.cuh"
#include "prep.cuh"
#include "resid.cuh"
#include "route.cuh"
#include "scan.cuh"

using namespace dsa;

namespace {

constexpr int kTargetCtas = 296;  // split-K decode: about two work items per SM (persistent CTAs)
constexpr size_t kAlign = 256;

inline size_t align_up(size_t x, size_t a = kAlign) { return (x + a - 1) / a * a; }

bool pow2_in(int v, int lo, int hi) { return v >= lo && v <= hi && (v & (v - 1)) == 0; }

// ------------------------------------------------------------- scan plan --
struct ScanPlan {
  MmaKind kind;
  bool split;
  int parts, esz, atoms, kstages, tstages, kt;
  int QG, G, qcols, stage_cols, n_qt, C, chunk, n_items, keep, nsub, capw;
  int rows;
  size_t smem;
  int ctas_per_sm;
};

constexpr size_t kSmemBudget = 227 * 1024;

// Dynamic shared memory of the scan: alignment slack, Q tiles, K stages of kt
// key tiles, then the per-row histograms (streaming rows) or the candidate
// array (gathered rows).
size_t scan_smem_bytes(MmaKind kind, int G, int QG, int qcols, int kstages, bool gather,
                       int kt = 1) {
  const int esz = kind == MmaKind::TF32 ? 4 : (kind == MmaKind::BF16 ? 2 : 1);
  const int atoms = esz;  // d = 128
  size_t q = align_up((size_t)G * atoms * qcols * 128, 1024);
  size_t k = (size_t)kstages * kt * atoms * 128 * 128;
  size_t h = gather ? (size_t)kMaxGatherKeys * sizeof(uint64_t) +
                          (size_t)kGatherBins * sizeof(uint32_t) +
                          (size_t)kGatherBoundary * sizeof(uint64_t)
                    : (size_t)G * QG * kHistWords * sizeof(uint32_t);
  return 1024 + q + k + h + sizeof(ScanSmemTail);
}

// Residency and pipeline depths of a planned scan: CTAs per SM from shared
// memory and TMEM; a CTA alone on its SM deepens its K pipeline into the
// spare shared memory, and the TMEM accumulator stages fill 512 columns.
void finish_plan(ScanPlan& pl, bool gather) {
  pl.smem = scan_smem_bytes(pl.kind, pl.G, pl.QG, pl.qcols, pl.kstages, gather, pl.kt);
  // 320 threads at up to 168 registers take more than half the register file:
  // one CTA per SM, whatever shared memory and TMEM would allow
  pl.ctas_per_sm = 1;
  {
    while (pl.kstages < 6 &&
           scan_smem_bytes(pl.kind, pl.G, pl.QG, pl.qcols, pl.kstages + 1, gather, pl.kt) <=
               kSmemBudget)
      ++pl.kstages;
    pl.smem = scan_smem_bytes(pl.kind, pl.G, pl.QG, pl.qcols, pl.kstages, gather, pl.kt);
  }
  pl.tstages = 512 / (pl.ctas_per_sm * pl.stage_cols);
  if (pl.tstages > kMaxTStages) pl.tstages = kMaxTStages;
  if (pl.tstages < 2) pl.tstages = 2;
}

// H: heads scanned; n_q / n_k / batch: geometry; keep: entries kept per row.
ScanPlan plan_scan(MmaKind kind, bool split, int batch, int n_q, int n_k, int H, int keep) {
  ScanPlan pl{};
  pl.kind = kind;
  pl.split = split;
  pl.parts = split ? 2 : 1;
  pl.esz = kind == MmaKind::TF32 ? 4 : (kind == MmaKind::BF16 ? 2 : 1);
  pl.atoms = pl.esz;
  pl.kstages = kind == MmaKind::E4M3 ? 4 : 2;
  const int ncols_max = kind == MmaKind::TF32 ? 128 : 256;
  const int hp = H * pl.parts;
  int QG = ncols_max / hp;
  const int qg_min = hp >= 16 ? 1 : 16 / hp;
  while (QG > qg_min && QG / 2 >= n_q) QG /= 2;  // few query rows (decode): shrink
  int G = (kind == MmaKind::TF32 || QG == 1 || n_q <= QG) ? 1 : 2;
#ifdef DSA_ONE_GROUP
  G = 1;
#endif
  // fit the shared-memory budget and the per-item row limit
  while (G * QG > kMaxRows ||
         scan_smem_bytes(kind, G, QG, QG * hp, pl.kstages, false) > kSmemBudget) {
    if (G == 2) G = 1;
    else if (QG > qg_min) QG /= 2;
    else break;
  }
  pl.QG = QG;
  pl.G = G;
  pl.qcols = QG * hp;
  // one e4m3 query row per item (decode): two 128-key tiles per K stage and per
  // accumulator hand-off, which halves the per-key count of pipeline hand-offs
  pl.kt = (kind == MmaKind::E4M3 && G == 1 && QG == 1 && H <= 64) ? 2 : 1;
  {
    const int n = QG * H * pl.kt;  // MMA N (the split-query parts share one
                                   // accumulator) times the key tiles of a unit
    pl.stage_cols = n > 128 ? 256 : (n > 64 ? 128 : 64);
  }
  pl.n_qt = (n_q + QG * G - 1) / (QG * G);
  pl.rows = batch * n_q;
  finish_plan(pl, false);
  pl.nsub = QG == 1 ? 8 : 4;
  // split-K over keys when there are too few query tiles to fill the GPU
  const long long tiles = (long long)batch * pl.n_qt;
  int C = 1, chunk = 0;
  if (tiles < kTargetCtas && n_k > 4 * 128) {
    C = (int)(kTargetCtas / tiles);  // one round: batch * tiles * C <= target
    if (C < 1) C = 1;
    if (C * pl.nsub > kFinMaxSeg) C = kFinMaxSeg / pl.nsub;
    chunk = (n_k + C - 1) / C;
    chunk = (chunk + 127) / 128 * 128;
    if (chunk < 512) chunk = 512;
    C = (n_k + chunk - 1) / chunk;
    if (C <= 1) {
      C = 1;
      chunk = 0;
    }
  }
  pl.C = C;
  pl.chunk = chunk;
  pl.n_items = (int)(tiles * C);
  pl.keep = keep;
  pl.capw = 2 * keep + kCompactSlack + 128;
  return pl;
}

// Plan of a gathered-key scan: every query row has its own key list, so a work
// item is one row (QG = G = 1, no split-K) and the MMA N is its heads (at least 16).
ScanPlan plan_gather(MmaKind kind, int batch, int n_q, int H, int keep) {
  ScanPlan pl{};
  pl.kind = kind;
  pl.split = false;
  pl.parts = 1;
  pl.esz = kind == MmaKind::TF32 ? 4 : (kind == MmaKind::BF16 ? 2 : 1);
  pl.atoms = pl.esz;
  pl.kstages = 2;
  pl.kt = 1;
  pl.QG = 1;
  pl.G = 1;
  pl.qcols = H < 16 ? 16 : H;
  // narrow accumulators: more TMEM stages let the MMA run further ahead
  pl.stage_cols = pl.qcols > 128 ? 256 : (pl.qcols > 64 ? 128 : 64);
  pl.n_qt = n_q;
  pl.rows = batch * n_q;
  finish_plan(pl, true);
  // the row's exact top-keep is selected in the kernel: one sub-log of keep entries
  pl.nsub = 1;
  pl.C = 1;
  pl.chunk = 0;
  pl.n_items = batch * n_q;
  pl.keep = keep;
  pl.capw = keep;
  return pl;
}

// Log bytes of one planned stage (sub-logs, fills, thresholds).
size_t log_bytes(const ScanPlan& pl) {
  const size_t slots = (size_t)pl.rows * pl.C;
  return align_up(slots * pl.nsub * pl.capw * sizeof(uint64_t)) +
         align_up(slots * pl.nsub * sizeof(int32_t)) +
         align_up(slots * sizeof(unsigned long long));
}

// ---------------------------------------------------------- TMA encoding --
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D map over a row-major [rows, 128 elements] operand: box = 128 bytes x box_rows,
// 128-byte swizzle (the layout the MMA descriptors expect).
bool make_map(CUtensorMap* m, const void* base, int esz, uint64_t rows, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  CUtensorMapDataType dt = esz == 4   ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                           : esz == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                      : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  cuuint64_t dims[2] = {(cuuint64_t)(128), (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)128 * esz};
  cuuint32_t box[2] = {(cuuint32_t)(128 / esz), box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D map over the query of sparse attention, [T][heads][576] bf16: box of 64
// dimensions x 128 head rows x one token, 128-byte swizzle; head rows past
// `heads` read as zeros.
bool make_map_q3d(CUtensorMap* m, const void* base, uint64_t tokens, uint64_t heads) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)kMlaDqk, (cuuint64_t)heads, (cuuint64_t)tokens};
  cuuint64_t strides[2] = {(cuuint64_t)kMlaDqk * 2, (cuuint64_t)heads * kMlaDqk * 2};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D map over the DoSA block ranges [batch * 2][nblk][256] bf16: box of 64
// dimensions x 32 blocks x one (sequence, hi / lo) plane, 128-byte swizzle;
// blocks past nblk read as zeros.
bool make_map_ranges(CUtensorMap* m, const void* base, uint64_t nblk, uint64_t batch) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {256, (cuuint64_t)nblk, (cuuint64_t)batch * 2};
  cuuint64_t strides[2] = {256 * 2, (cuuint64_t)nblk * 256 * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)kDosaBT, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D map over the cached latent rows [rows][576] bf16 for four-row gathers:
// a one-row-high box of 64 dimensions.
bool make_map_kv(CUtensorMap* m, const void* base, uint64_t rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)kMlaDqk, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)kMlaDqk * 2};
  cuuint32_t box[2] = {64, 1};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <MmaKind K, bool S, int HT, int GATHER = 0, bool DOSA = false>
cudaError_t launch_scan_t(const ScanPlan& pl, const CUtensorMap& qm, const CUtensorMap& km,
                          const ScanArgs& a, cudaStream_t st) {
  auto kern = scan_kernel<K, S, HT, GATHER, DOSA>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)pl.smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int grid = sms * pl.ctas_per_sm;
  if (grid > pl.n_items) grid = pl.n_items;
  if (grid < 1) grid = 1;
  kern<<<grid, kScanThreads, pl.smem, st>>>(qm, km, a);
  return cudaGetLastError();
}

template <MmaKind K, bool S>
cudaError_t launch_scan_h(const ScanPlan& pl, const CUtensorMap& qm, const CUtensorMap& km,
                          const ScanArgs& a, cudaStream_t st) {
  switch (a.H) {
    case 8: return launch_scan_t<K, S, 8>(pl, qm, km, a, st);
    case 16: return launch_scan_t<K, S, 16>(pl, qm, km, a, st);
    case 32: return launch_scan_t<K, S, 32>(pl, qm, km, a, st);
    case 64: return launch_scan_t<K, S, 64>(pl, qm, km, a, st);
    default: return launch_scan_t<K, S, 128>(pl, qm, km, a, st);
  }
}

template <int GATHER>
cudaError_t launch_scan_gather(const ScanPlan& pl, const CUtensorMap& qm, const CUtensorMap& km,
                               const ScanArgs& a, cudaStream_t st) {
  switch (a.H) {  // routed / reranked stages run on bf16 operands
    case 8: return launch_scan_t<MmaKind::BF16, false, 8, GATHER>(pl, qm, km, a, st);
    case 16: return launch_scan_t<MmaKind::BF16, false, 16, GATHER>(pl, qm, km, a, st);
    case 32: return launch_scan_t<MmaKind::BF16, false, 32, GATHER>(pl, qm, km, a, st);
    case 64: return launch_scan_t<MmaKind::BF16, false, 64, GATHER>(pl, qm, km, a, st);
    default: return launch_scan_t<MmaKind::BF16, false, 128, GATHER>(pl, qm, km, a, st);
  }
}

cudaError_t launch_scan(const ScanPlan& pl, const CUtensorMap& qm, const CUtensorMap& km,
                        const ScanArgs& a, cudaStream_t st, int gather = 0) {
  if (gather == 1) return launch_scan_gather<1>(pl, qm, km, a, st);
  if (gather == 2) return launch_scan_gather<2>(pl, qm, km, a, st);
  if (a.dosa_ub != nullptr) {  // bound pruning: bf16 operands, heads >= 32 (validated)
    switch (a.H) {
      case 32: return launch_scan_t<MmaKind::BF16, false, 32, 0, true>(pl, qm, km, a, st);
      case 64: return launch_scan_t<MmaKind::BF16, false, 64, 0, true>(pl, qm, km, a, st);
      default: return launch_scan_t<MmaKind::BF16, false, 128, 0, true>(pl, qm, km, a, st);
    }
  }
  switch (pl.kind) {
    case MmaKind::TF32: return launch_scan_h<MmaKind::TF32, false>(pl, qm, km, a, st);
    case MmaKind::BF16: return launch_scan_h<MmaKind::BF16, false>(pl, qm, km, a, st);
    default:
      if (pl.split) {
        switch (a.H) {  // split-query path: heads >= 32
          case 32: return launch_scan_t<MmaKind::E4M3, true, 32>(pl, qm, km, a, st);
          case 64: return launch_scan_t<MmaKind::E4M3, true, 64>(pl, qm, km, a, st);
          default: return launch_scan_t<MmaKind::E4M3, true, 128>(pl, qm, km, a, st);
        }
      }
      return launch_scan_h<MmaKind::E4M3, false>(pl, qm, km, a, st);
  }
}

template <int NT, int E>
cudaError_t launch_fin(const FinalArgs& f, int groups, int stage_cap, size_t smem, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(finalize_kernel<NT, E>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  finalize_kernel<NT, E><<<(f.rows + groups - 1) / groups, NT * groups, smem, st>>>(f, groups,
                                                                                  stage_cap);
  return cudaGetLastError();
}

// Output mapping of a finalize call: row i of sequence b (of nq_c rows per
// sequence in the logs) is written at row b * nq_total + q_off + i.
struct OutMap {
  int nq_c, nq_total, q_off;
};

cudaError_t launch_finalize(const ScanPlan& pl, int topk, int sorted, const uint64_t* logs,
                            const int32_t* cnt, const unsigned long long* thr, int32_t* out_idx,
                            float* out_score, OutMap om, const int32_t* status, cudaStream_t st) {
  FinalArgs f{};
  f.rows = pl.rows;
  f.nq_c = om.nq_c;
  f.nq_total = om.nq_total;
  f.q_off = om.q_off;
  f.C = pl.C;
  f.nsub = pl.nsub;
  f.topk = topk;
  f.capw = pl.capw;
  int sc = pl.C == 1 ? 256 : 1024;  // at least one key per thread of a row group
  while (sc < topk) sc <<= 1;
  f.sort_cap = sc;
  f.sorted = sorted;
  f.logs = logs;
  f.log_cnt = cnt;
  f.log_thr = thr;
  f.out_idx = out_idx;
  f.out_score = out_score;
  f.status = status;
  if (pl.C == 1 && sc <= 2048) {
    // one key chunk per row: about k candidates; up to four rows per CTA
    const int stage_cap = sc + sc / 2;
    const size_t per_group = ((size_t)sc + stage_cap + kFinBoundary) * sizeof(uint64_t);
    const int e_per = sc / 256;
    int groups = (int)((160 * 1024) / per_group);
    if (groups > kFinMaxGroups) groups = kFinMaxGroups;
    if (groups < 1) groups = 1;
    const size_t smem = per_group * groups;
    switch (e_per) {
      case 1: return launch_fin<256, 1>(f, groups, stage_cap, smem, st);
      case 2: return launch_fin<256, 2>(f, groups, stage_cap, smem, st);
      case 4: return launch_fin<256, 4>(f, groups, stage_cap, smem, st);
      default: return launch_fin<256, 8>(f, groups, stage_cap, smem, st);
    }
  }
  // split-K rows (about C * k candidates) and large k: one row per 1024-thread CTA
  const size_t budget = 200 * 1024;
  int stage_cap = (int)(budget / sizeof(uint64_t)) - sc - kFinBoundary;
  if (stage_cap < sc) stage_cap = sc;
  const size_t smem = ((size_t)sc + stage_cap + kFinBoundary) * sizeof(uint64_t);
  switch (sc / 1024) {
    case 1: return launch_fin<1024, 1>(f, 1, stage_cap, smem, st);
    case 2: return launch_fin<1024, 2>(f, 1, stage_cap, smem, st);
    case 4: return launch_fin<1024, 4>(f, 1, stage_cap, smem, st);
    default: return launch_fin<1024, 8>(f, 1, stage_cap, smem, st);
  }
}

// Device-side input checks under DSA_FLAG_CHECK: scales finite and positive,
// lengths inside [0, n_k].
__global__ void check_inputs_kernel(const float* qs, int64_t nqs, const float* ks, int64_t nks,
                                    const int32_t* pos0, const int32_t* klen, int batch, int n_k,
                                    int32_t* status) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t j = i; j < nqs; j += stride)
    if (!(isfinite(qs[j]) && qs[j] > 0.f)) set_status(status, DSA_ERR_NONFINITE, 100);
  for (int64_t j = i; j < nks; j += stride)
    if (!(isfinite(ks[j]) && ks[j] > 0.f)) set_status(status, DSA_ERR_NONFINITE, 101);
  for (int64_t j = i; j < batch; j += stride) {
    if (klen && (klen[j] < 0 || klen[j] > n_k)) set_status(status, DSA_ERR_INVALID, 102);
    if (pos0 && pos0[j] < 0) set_status(status, DSA_ERR_INVALID, 103);
  }
}

// ------------------------------------------------------------ validation --
int validate_problem(const dsa_problem* p) {
  if (!p) return DSA_ERR_INVALID;
  if (p->batch < 1 || p->n_q < 1 || p->n_k < 1 || p->heads < 1 || p->dim < 1 || p->topk < 1)
    return DSA_ERR_INVALID;
  if (p->dim != 128) return DSA_ERR_UNSUPPORTED;
  if (!pow2_in(p->heads, 8, 128)) return DSA_ERR_UNSUPPORTED;
  if (p->topk > 8192) return DSA_ERR_UNSUPPORTED;
  if (p->n_k > (1 << 24) || (long long)p->batch * p->n_k > (1ll << 31)) return DSA_ERR_UNSUPPORTED;
  if ((long long)p->batch * p->n_q * p->heads * 2 > (1ll << 31)) return DSA_ERR_UNSUPPORTED;
  const int qd = p->q_dtype, kd = p->k_dtype;
  if (qd < DSA_F32 || qd > DSA_E4M3 || kd < DSA_F32 || kd > DSA_E4M3) return DSA_ERR_INVALID;
  const bool same = qd == kd;
  const bool split = (qd == DSA_BF16 || qd == DSA_F32) && kd == DSA_E4M3;
  if (!same && !split) return DSA_ERR_UNSUPPORTED;
  if (split && p->heads < 32) return DSA_ERR_UNSUPPORTED;
  if ((p->flags & DSA_FLAG_SORTED) && (p->flags & DSA_FLAG_BY_POSITION)) return DSA_ERR_INVALID;
  if ((p->flags & DSA_FLAG_DOSA) && !(qd == DSA_BF16 && kd == DSA_BF16 && p->heads >= 32))
    return DSA_ERR_UNSUPPORTED;
  return DSA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// Output order of a problem: 0 any, 1 (score desc, index asc), 2 index asc.
int out_order(const dsa_problem* p) {
  if (p->flags & DSA_FLAG_BY_POSITION) return 2;
  return (p->flags & DSA_FLAG_SORTED) ? 1 : 0;
}

// Kind / split decision of a validated problem.
void kind_of(const dsa_problem* p, MmaKind* kind, bool* split) {
  *split = (p->q_dtype != DSA_E4M3) && p->k_dtype == DSA_E4M3;
  if (p->k_dtype == DSA_E4M3)
    *kind = MmaKind::E4M3;
  else if (p->k_dtype == DSA_BF16)
    *kind = MmaKind::BF16;
  else
    *kind = MmaKind::TF32;
}

// DoSA bound blocks: 2^kDosaShift tokens (a whole number of 128-key tiles).
constexpr int kDosaShift = 10;

struct DsaLayout {
  ScanPlan pl;
  size_t off_logs, off_cnt, off_thr, off_parts, off_hscale;
  size_t off_ranges, off_mx, off_ub, off_lb, off_seed;  // DoSA (DSA_FLAG_DOSA) only
  int dosa_nblk;
  size_t total;
};

DsaLayout dsa_layout(const dsa_problem* p) {
  DsaLayout L{};
  MmaKind kind;
  bool split;
  kind_of(p, &kind, &split);
  L.pl = plan_scan(kind, split, p->batch, p->n_q, p->n_k, p->heads, p->topk);
  size_t off = kWsHeaderBytes;
  const size_t slots = (size_t)L.pl.rows * L.pl.C;
  L.off_logs = off;
  off += align_up(slots * L.pl.nsub * L.pl.capw * sizeof(uint64_t));
  L.off_cnt = off;
  off += align_up(slots * L.pl.nsub * sizeof(int32_t));
  L.off_thr = off;
  off += align_up(slots * sizeof(unsigned long long));
  L.off_parts = off;
  if (split) off += align_up((size_t)L.pl.rows * 2 * p->heads * p->dim);
  L.off_hscale = off;
  if (split) off += align_up((size_t)L.pl.rows * p->heads * sizeof(float));
  L.off_ranges = L.off_mx = L.off_ub = L.off_lb = L.off_seed = off;
  L.dosa_nblk = 0;
  if (p->flags & DSA_FLAG_DOSA) {
    L.dosa_nblk = (p->n_k + (1 << kDosaShift) - 1) >> kDosaShift;
    off += align_up((size_t)p->batch * 2 * L.dosa_nblk * 256 * 2);
    L.off_mx = off;
    off += align_up((size_t)p->batch * L.dosa_nblk * sizeof(float));
    L.off_ub = off;
    off += align_up((size_t)p->batch * p->n_q * L.dosa_nblk * sizeof(float));
    L.off_lb = off;
    off += align_up((size_t)p->batch * p->n_q * L.dosa_nblk * sizeof(float));
    L.off_seed = off;
    off += align_up((size_t)p->batch * p->n_q * sizeof(float));
  }
  L.total = off;
  return L;
}

int finish(const dsa_problem* p, void* ws, cudaStream_t st) {
  if (cudaPeekAtLastError() != cudaSuccess) {
    cudaGetLastError();
    return DSA_ERR_CUDA;
  }
  if (p->flags & DSA_FLAG_CHECK) return dsa_read_status(ws, st);
  return DSA_OK;
}

// ----------------------------------------------------- allocation-free path --
// Scratch of dsa_index_noalloc: a fixed 64 MiB array in device memory that
// every GPU loading this library holds until the process exits.  Host code
// must not use the name as an address; the device address comes from
// cudaGetSymbolAddress, taken once per device with that device current and
// kept for the life of the process (a cudaDeviceReset would reload the module
// and could move it; the header rules that use out).
constexpr size_t kNoAllocScratchBytes = 64ull << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_addr[kNoAllocMaxDevices];  // per-device address, null until set up

int noalloc_scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoAllocMaxDevices) {
    cudaGetLastError();
    return DSA_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return DSA_ERR_CUDA;
    }
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return DSA_OK;
}

// ------------------------------------------------------------- routed paths --
// MISA, MISA-dagger and HISA chain scan stages over row chunks: every stage of
// a chunk writes candidate logs into one shared log region, so the workspace
// holds the logs of one chunk, bounded by kRouteLogBudget.
constexpr size_t kRouteLogBudget = 8ull << 30;

int log2_exact(int v) {
  int s = 0;
  while ((1 << s) < v) ++s;
  return s;
}

struct RouteCfg {
  int algo;
  bool route;        // the MISA router runs (MISA, MISA-dagger, stacked HISA)
  int h, bsR, nblkR, ncolsR;
  bool hisa;
  int bsH, nblkH, r;
  int kp;            // MISA-dagger / LISA-dagger pool size
  int hh;            // heads of the token stages
  int list_len;      // per-row list of the second stage (pool or blocks), 0 for MISA
  bool pseudo;       // LISA / ResMiSA: the token stage runs on pseudo-head rows
  int hp;            // pseudo-heads per row (power of two >= 4 + res_r)
  bool res;          // ResMiSA: the residual router runs
  int bsX, nblkX, res_r;  // ResMiSA router block shift, full blocks, residual heads
};

int route_cfg(const dsa_problem* p, int algo, const dsa_route_params* rp, RouteCfg* c) {
  if (!rp) return DSA_ERR_INVALID;
  if (algo != DSA_ALGO_MISA && algo != DSA_ALGO_MISA_DAGGER && algo != DSA_ALGO_HISA &&
      algo != DSA_ALGO_LISA && algo != DSA_ALGO_RESMISA)
    return DSA_ERR_INVALID;
  if (p->q_dtype != DSA_BF16 || p->k_dtype != DSA_BF16) return DSA_ERR_UNSUPPORTED;
  if (p->batch > 65535) return DSA_ERR_UNSUPPORTED;
  if (p->flags & DSA_FLAG_DOSA) return DSA_ERR_UNSUPPORTED;  // bounds of the dense scan only
  *c = RouteCfg{};
  c->algo = algo;
  if (algo == DSA_ALGO_LISA || algo == DSA_ALGO_RESMISA) {
    c->pseudo = true;
    if (algo == DSA_ALGO_LISA) {
      c->hp = 8;
      if (rp->lisa_pool != 0) {
        if (rp->lisa_pool < p->topk) return DSA_ERR_INVALID;
        if (rp->lisa_pool > 8192) return DSA_ERR_UNSUPPORTED;
        c->kp = rp->lisa_pool;
        c->list_len = c->kp;
      }
    } else {
      if (rp->res_r < 0 || rp->res_r > p->heads) return DSA_ERR_INVALID;
      if (rp->res_r > 124) return DSA_ERR_UNSUPPORTED;
      if (!pow2_in(rp->res_block, 16, 4096)) return DSA_ERR_UNSUPPORTED;
      c->res = true;
      c->res_r = rp->res_r;
      c->bsX = log2_exact(rp->res_block);
      c->nblkX = p->n_k >> c->bsX;
      c->hp = 8;
      while (c->hp < 4 + c->res_r) c->hp *= 2;
    }
    c->hh = c->hp;
    return DSA_OK;
  }
  c->route = algo != DSA_ALGO_HISA || rp->misa_h > 0;
  if (c->route) {
    if (rp->misa_h < 1 || rp->misa_h > p->heads) return DSA_ERR_INVALID;
    if (!pow2_in(rp->misa_h, 8, 128)) return DSA_ERR_UNSUPPORTED;
    if (!pow2_in(rp->misa_block, 16, 4096)) return DSA_ERR_UNSUPPORTED;
    c->h = rp->misa_h;
    c->bsR = log2_exact(rp->misa_block);
    c->nblkR = p->n_k >> c->bsR;
    if (c->nblkR > kRouterBColsMax) return DSA_ERR_UNSUPPORTED;
    c->ncolsR = c->nblkR <= 16 ? 16 : (c->nblkR + 15) / 16 * 16;
  }
  if (algo == DSA_ALGO_MISA_DAGGER) {
    if (rp->k_prime < p->topk) return DSA_ERR_INVALID;
    if (rp->k_prime > 8192) return DSA_ERR_UNSUPPORTED;
    c->kp = rp->k_prime;
    c->list_len = c->kp;
  }
  if (algo == DSA_ALGO_HISA) {
    if (!pow2_in(rp->hisa_block, 16, 4096)) return DSA_ERR_UNSUPPORTED;
    if (rp->hisa_r < 1) return DSA_ERR_INVALID;
    if (rp->hisa_r > 8192) return DSA_ERR_UNSUPPORTED;
    c->hisa = true;
    c->bsH = log2_exact(rp->hisa_block);
    c->nblkH = p->n_k >> c->bsH;
    c->r = rp->hisa_r;
    c->list_len = c->r;
    if (((long long)c->r << c->bsH) > kMaxGatherKeys) return DSA_ERR_UNSUPPORTED;
  }
  c->hh = c->route ? c->h : p->heads;
  return DSA_OK;
}

// Stage plans of one chunk of nq query rows per sequence.
struct RouteStages {
  ScanPlan s1;  // MISA: routed scan; MISA-dagger: routed scan keeping k'; HISA: coarse block scan
  ScanPlan s2;  // MISA-dagger: rerank of the pool; HISA: rerank of the kept blocks' tokens
  bool two;
};

RouteStages plan_route(const dsa_problem* p, const RouteCfg& c, int nq) {
  RouteStages rs{};
  if (c.pseudo) {
    // the pseudo-head scan keeps the LISA-dagger pool or the final top-k
    rs.s1 = plan_scan(MmaKind::BF16, false, p->batch, nq, p->n_k, c.hp, c.kp > 0 ? c.kp : p->topk);
    if (c.kp > 0) {
      rs.s2 = plan_gather(MmaKind::BF16, p->batch, nq, p->heads, p->topk);
      rs.two = true;
    }
  } else if (c.algo == DSA_ALGO_MISA) {
    rs.s1 = plan_scan(MmaKind::BF16, false, p->batch, nq, p->n_k, c.h, p->topk);
  } else if (c.algo == DSA_ALGO_MISA_DAGGER) {
    rs.s1 = plan_scan(MmaKind::BF16, false, p->batch, nq, p->n_k, c.h, c.kp);
    rs.s2 = plan_gather(MmaKind::BF16, p->batch, nq, p->heads, p->topk);
    rs.two = true;
  } else {
    rs.s1 = plan_scan(MmaKind::BF16, false, p->batch, nq, c.nblkH > 0 ? c.nblkH : 1, c.hh, c.r);
    rs.s2 = plan_gather(MmaKind::BF16, p->batch, nq, c.hh, p->topk);
    rs.two = true;
  }
  return rs;
}

size_t stages_log_bytes(const RouteStages& rs) {
  size_t b = log_bytes(rs.s1);
  if (rs.two) {
    const size_t b2 = log_bytes(rs.s2);
    if (b2 > b) b = b2;
  }
  return b;
}

struct RouteLayout {
  RouteCfg c;
  int nq_c, n_chunks;
  size_t fullR_rows, fullH_rows;
  size_t off_runR, off_fullR, off_heads, off_qg, off_wg, off_runH, off_fullH, off_list, off_logs;
  size_t off_extrun, off_extfull;
  size_t total;
};

RouteLayout route_layout(const dsa_problem* p, const RouteCfg& c) {
  RouteLayout L{};
  L.c = c;
  const size_t rows = (size_t)p->batch * p->n_q;
  // row chunk: halve until the candidate logs of one chunk fit the budget
  int nq = p->n_q;
  while (nq > 16 && stages_log_bytes(plan_route(p, c, nq)) > kRouteLogBudget) nq = (nq + 1) / 2;
  L.nq_c = nq;
  L.n_chunks = (p->n_q + nq - 1) / nq;
  size_t logs = stages_log_bytes(plan_route(p, c, nq));
  const int last = p->n_q - (L.n_chunks - 1) * nq;  // a short last chunk may split keys more
  const size_t logs_last = stages_log_bytes(plan_route(p, c, last));
  if (logs_last > logs) logs = logs_last;
  size_t off = kWsHeaderBytes;
  if (c.pseudo) {
    L.off_qg = off;
    off += align_up(rows * c.hp * 128 * 2);
    L.off_wg = off;
    off += align_up(rows * c.hp * sizeof(float));
  }
  if (c.res) {
    L.off_extrun = off;
    off += align_up((size_t)p->batch * p->n_k * 256 * 2);
    L.off_extfull = off;
    off += align_up((size_t)p->batch * (c.nblkX > 0 ? c.nblkX : 1) * 256 * 2);
    L.off_heads = off;
    off += align_up(rows * (c.res_r > 0 ? c.res_r : 1) * sizeof(int32_t));
  }
  if (c.route) {
    L.fullR_rows = (size_t)p->batch * (c.nblkR > 0 ? c.nblkR : 1) + 256;
    L.off_runR = off;
    off += align_up((size_t)p->batch * p->n_k * 128 * 2);
    L.off_fullR = off;
    off += align_up(L.fullR_rows * 128 * 2);
    L.off_heads = off;
    off += align_up(rows * c.h * sizeof(int32_t));
    L.off_qg = off;
    off += align_up(rows * c.h * 128 * 2);
    L.off_wg = off;
    off += align_up(rows * c.h * sizeof(float));
  }
  if (c.hisa) {
    L.fullH_rows = (size_t)p->batch * (c.nblkH > 0 ? c.nblkH : 1) + 128;
    L.off_runH = off;
    off += align_up((size_t)p->batch * p->n_k * 128 * 2);
    L.off_fullH = off;
    off += align_up(L.fullH_rows * 128 * 2);
  }
  L.off_list = off;
  off += align_up((size_t)p->batch * nq * c.list_len * sizeof(int32_t));
  L.off_logs = off;
  off += logs;
  L.total = off;
  return L;
}

struct LogPtrs {
  uint64_t* logs;
  int32_t* cnt;
  unsigned long long* thr;
};

LogPtrs log_ptrs(const ScanPlan& pl, uint8_t* base) {
  const size_t slots = (size_t)pl.rows * pl.C;
  LogPtrs lp;
  lp.logs = reinterpret_cast<uint64_t*>(base);
  base += align_up(slots * pl.nsub * pl.capw * sizeof(uint64_t));
  lp.cnt = reinterpret_cast<int32_t*>(base);
  base += align_up(slots * pl.nsub * sizeof(int32_t));
  lp.thr = reinterpret_cast<unsigned long long*>(base);
  return lp;
}

// Operands of one bf16 scan stage.
struct StageIO {
  const void* q;          // [batch, q_stride, H, 128]
  const float* w;         // [batch, q_stride, H]
  int q_stride, H;
  const void* k;          // key map rows (tokens or block representatives)
  uint64_t k_rows;        // rows of the key map
  uint32_t k_box;         // TMA box height of the key map
  int n_kmap;             // key rows per sequence in the key map
  int bs_shift;           // > 0: keys are full-block representatives
  const int32_t* klist;   // gathered stages: per-row lists
  int klist_len, lb_shift, gather;
};

int run_stage(const dsa_problem* p, const ScanPlan& pl, const StageIO& io, int q_off, int nq,
              const LogPtrs& lp, int32_t* status, cudaStream_t st) {
  CUtensorMap qm, km;
  if (!make_map(&qm, io.q, 2, (uint64_t)p->batch * io.q_stride * io.H, (uint32_t)pl.qcols))
    return DSA_ERR_CUDA;
  if (!make_map(&km, io.k, 2, io.k_rows, io.k_box)) return DSA_ERR_CUDA;
  ScanArgs a{};
  a.batch = p->batch;
  a.n_q = nq;
  a.n_k = io.n_kmap;
  a.H = io.H;
  a.d = p->dim;
  a.q_stride = io.q_stride;
  a.q_off = q_off;
  a.n_tok = p->n_k;
  a.bs_shift = io.bs_shift;
  a.klist = io.klist;
  a.klist_len = io.klist_len;
  a.kraw = reinterpret_cast<const uint16_t*>(io.k);
  a.lb_shift = io.lb_shift;
  a.keep = pl.keep;
  a.QG = pl.QG;
  a.qcols = pl.qcols;
  a.kstages = pl.kstages;
  a.kt = pl.kt;
  a.tstages = pl.tstages;
  a.G = pl.G;
  a.stage_cols = pl.stage_cols;
  a.n_qt = pl.n_qt;
  a.C = pl.C;
  a.chunk = pl.chunk;
  a.n_items = pl.n_items;
  a.q_pos0 = p->q_pos0;
  a.k_len = p->k_len;
  a.w = io.w;
  a.nsub = pl.nsub;
  a.capw = pl.capw;
  a.logs = lp.logs;
  a.log_cnt = lp.cnt;
  a.log_thr = lp.thr;
  a.status = status;
  a.wait_cycles = kWaitCycles;
  a.test_stall = 0;
  return launch_scan(pl, qm, km, a, st, io.gather) == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

int launch_pool(const void* k, const dsa_problem* p, int bs_shift, uint8_t* run, uint8_t* full,
                int nblk, cudaStream_t st) {
  const int nb = (p->n_k + (1 << bs_shift) - 1) >> bs_shift;
  pool_prefix_kernel<false><<<dim3((unsigned)nb, (unsigned)p->batch), 128, 0, st>>>(
      k, p->n_k, bs_shift, run, full, nblk);
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

template <int H>
cudaError_t launch_router_h(const CUtensorMap& am, const CUtensorMap& bm, const CUtensorMap& rm,
                            const RouterArgs& a, cudaStream_t st) {
  const int smem = (int)router_smem_bytes();
  cudaError_t e =
      cudaFuncSetAttribute(router_kernel<H>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int grid = a.n_tiles < sms ? a.n_tiles : sms;
  if (grid < 1) grid = 1;
  router_kernel<H><<<grid, kRouterThreads, smem, st>>>(am, bm, rm, a);
  return cudaGetLastError();
}

// Pooling + router: heads, optional E, gathered q / w rows of every query.
int run_router(const dsa_problem* p, const RouteLayout& L, const void* q, const void* k,
               const float* w, int32_t* heads, float* E, uint8_t* ws, cudaStream_t st) {
  const RouteCfg& c = L.c;
  uint8_t* runR = ws + L.off_runR;
  uint8_t* fullR = ws + L.off_fullR;
  int rc = launch_pool(k, p, c.bsR, runR, fullR, c.nblkR, st);
  if (rc != DSA_OK) return rc;
  CUtensorMap am, bm, rm;
  if (!make_map(&am, q, 2, (uint64_t)p->batch * p->n_q * p->heads, 128)) return DSA_ERR_CUDA;
  if (!make_map(&bm, fullR, 2, L.fullR_rows, (uint32_t)c.ncolsR)) return DSA_ERR_CUDA;
  if (!make_map(&rm, runR, 2, (uint64_t)p->batch * p->n_k, 1)) return DSA_ERR_CUDA;
  RouterArgs a{};
  a.batch = p->batch;
  a.n_q = p->n_q;
  a.n_tok = p->n_k;
  a.H = p->heads;
  a.h = c.h;
  a.bs_shift = c.bsR;
  a.nblk = c.nblkR;
  a.ncols = c.ncolsR;
  a.tiles_per_seq = (p->n_q * p->heads + 127) / 128;
  a.n_tiles = p->batch * a.tiles_per_seq;
  a.q_pos0 = p->q_pos0;
  a.k_len = p->k_len;
  a.q = reinterpret_cast<const uint16_t*>(q);
  a.w = w;
  a.heads = heads;
  a.E = E;
  a.qg = reinterpret_cast<uint16_t*>(ws + L.off_qg);
  a.wg = reinterpret_cast<float*>(ws + L.off_wg);
  a.status = reinterpret_cast<int32_t*>(ws);
  cudaError_t e;
  switch (p->heads) {
    case 8: e = launch_router_h<8>(am, bm, rm, a, st); break;
    case 16: e = launch_router_h<16>(am, bm, rm, a, st); break;
    case 32: e = launch_router_h<32>(am, bm, rm, a, st); break;
    case 64: e = launch_router_h<64>(am, bm, rm, a, st); break;
    default: e = launch_router_h<128>(am, bm, rm, a, st); break;
  }
  return e == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

// Copy a chunk's per-row lists [batch, nq, len] into rows q_off.. of out [batch, n_q, len].
int copy_lists(int32_t* out, const int32_t* lists, const dsa_problem* p, int q_off, int nq,
               int len, cudaStream_t st) {
  const size_t row = (size_t)len * sizeof(int32_t);
  return cudaMemcpy2DAsync(out + (size_t)q_off * len, (size_t)p->n_q * row, lists, (size_t)nq * row,
                           (size_t)nq * row, (size_t)p->batch, cudaMemcpyDeviceToDevice,
                           st) == cudaSuccess
             ? DSA_OK
             : DSA_ERR_CUDA;
}

// Shared set-up of the routed entry points: validation, layout, status reset,
// optional device checks.
int route_begin(const dsa_problem* p, int algo, const dsa_route_params* rp, const void* q,
                const void* k, const float* w, int32_t* out_idx, float* out_score, void* ws,
                size_t ws_bytes, cudaStream_t st, RouteLayout* L) {
  int v = validate_problem(p);
  if (v != DSA_OK) return v;
  RouteCfg c;
  v = route_cfg(p, algo, rp, &c);
  if (v != DSA_OK) return v;
  if (!q || !k || !w || !out_idx || !out_score) return DSA_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k)) return DSA_ERR_INVALID;
  *L = route_layout(p, c);
  if (!ws || ws_bytes < L->total) return DSA_ERR_WORKSPACE;
  if (!aligned16(ws)) return DSA_ERR_INVALID;
  uint8_t* w8 = reinterpret_cast<uint8_t*>(ws);
  if (cudaMemsetAsync(w8, 0, kWsHeaderBytes, st) != cudaSuccess) return DSA_ERR_CUDA;
  if (p->flags & DSA_FLAG_CHECK)
    check_inputs_kernel<<<64, 256, 0, st>>>(nullptr, 0, nullptr, 0, p->q_pos0, p->k_len, p->batch,
                                            p->n_k, reinterpret_cast<int32_t*>(w8));
  return DSA_OK;
}

// Pseudo-head rows of every query (LISA: the linear term; ResMiSA: plus the
// residual heads), written into the workspace for the token scan.
int run_pseudo(const dsa_problem* p, const RouteLayout& L, const void* q, const float* w,
               const int32_t* heads, uint8_t* ws, cudaStream_t st) {
  PseudoArgs a{};
  a.rows = (int64_t)p->batch * p->n_q;
  a.H = p->heads;
  a.HP = L.c.hp;
  a.r = L.c.res_r;
  a.q = reinterpret_cast<const uint16_t*>(q);
  a.w = w;
  a.heads = heads;
  a.qp = reinterpret_cast<uint16_t*>(ws + L.off_qg);
  a.wp = reinterpret_cast<float*>(ws + L.off_wg);
  pseudo_heads_kernel<<<(unsigned)((a.rows + 7) / 8), 256, 0, st>>>(a);
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

// The pseudo-head token scan over every legal key, then (LISA-dagger) the
// all-head rerank of each row's pool; per row chunk.
int run_pseudo_stages(const dsa_problem* p, const RouteLayout& L, const void* q, const void* k,
                      const float* w, int32_t* out_idx, float* out_score, int32_t* out_pool,
                      uint8_t* ws, cudaStream_t st) {
  int32_t* status = reinterpret_cast<int32_t*>(ws);
  const int sorted = out_order(p);
  int32_t* pool = reinterpret_cast<int32_t*>(ws + L.off_list);
  for (int ci = 0; ci < L.n_chunks; ++ci) {
    const int q_off = ci * L.nq_c;
    const int nq = p->n_q - q_off < L.nq_c ? p->n_q - q_off : L.nq_c;
    const RouteStages rs = plan_route(p, L.c, nq);
    LogPtrs lp = log_ptrs(rs.s1, ws + L.off_logs);
    StageIO io{};
    io.q = ws + L.off_qg;
    io.w = reinterpret_cast<const float*>(ws + L.off_wg);
    io.q_stride = p->n_q;
    io.H = L.c.hp;
    io.k = k;
    io.k_rows = (uint64_t)p->batch * p->n_k;
    io.k_box = 128;
    io.n_kmap = p->n_k;
    int rc = run_stage(p, rs.s1, io, q_off, nq, lp, status, st);
    if (rc != DSA_OK) return rc;
    if (L.c.kp == 0) {
      if (launch_finalize(rs.s1, p->topk, sorted, lp.logs, lp.cnt, lp.thr, out_idx, out_score,
                          OutMap{nq, p->n_q, q_off}, status, st) != cudaSuccess)
        return DSA_ERR_CUDA;
      continue;
    }
    if (launch_finalize(rs.s1, L.c.kp, 0, lp.logs, lp.cnt, lp.thr, pool, nullptr,
                        OutMap{nq, nq, 0}, status, st) != cudaSuccess)
      return DSA_ERR_CUDA;
    if (out_pool) {
      rc = copy_lists(out_pool, pool, p, q_off, nq, L.c.kp, st);
      if (rc != DSA_OK) return rc;
    }
    lp = log_ptrs(rs.s2, ws + L.off_logs);
    StageIO io2{};
    io2.q = q;
    io2.w = w;
    io2.q_stride = p->n_q;
    io2.H = p->heads;
    io2.k = k;
    io2.k_rows = (uint64_t)p->batch * p->n_k;
    io2.k_box = 1;
    io2.n_kmap = p->n_k;
    io2.klist = pool;
    io2.klist_len = L.c.kp;
    io2.gather = 1;
    rc = run_stage(p, rs.s2, io2, q_off, nq, lp, status, st);
    if (rc != DSA_OK) return rc;
    if (launch_finalize(rs.s2, p->topk, sorted, lp.logs, lp.cnt, lp.thr, out_idx, out_score,
                        OutMap{nq, p->n_q, q_off}, status, st) != cudaSuccess)
      return DSA_ERR_CUDA;
  }
  return DSA_OK;
}

}  // namespace

// ===================================================================== ABI ==
extern "C" {

const char* dsa_status_string(int32_t s) {
  switch (s) {
    case DSA_OK: return "ok";
    case DSA_ERR_INVALID: return "invalid argument (null pointer, bad size or inconsistent shape)";
    case DSA_ERR_UNSUPPORTED: return "unsupported dtype, dim, heads or top-k";
    case DSA_ERR_WORKSPACE: return "workspace missing or smaller than dsa_workspace_size()";
    case DSA_ERR_CUDA: return "CUDA runtime error or launch failure";
    case DSA_ERR_NONFINITE: return "non-finite, zero or negative scale";
    case DSA_ERR_TIMEOUT: return "a bounded device wait expired";
    case DSA_ERR_INTERNAL: return "a device-side capacity or bounds check failed";
    default: return "unknown status";
  }
}

int dsa_read_status(const void* workspace, void* stream) {
  if (!workspace) return DSA_ERR_INVALID;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return DSA_ERR_CUDA;
  int32_t s = 0;
  if (cudaMemcpy(&s, workspace, sizeof(s), cudaMemcpyDeviceToHost) != cudaSuccess)
    return DSA_ERR_CUDA;
  return s;
}

int dsa_read_pruned(const void* workspace, void* stream, unsigned long long* pruned) {
  if (!workspace || !pruned) return DSA_ERR_INVALID;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return DSA_ERR_CUDA;
  if (cudaMemcpy(pruned, reinterpret_cast<const uint8_t*>(workspace) + offsetof(WsHeader, pruned),
                 sizeof(*pruned), cudaMemcpyDeviceToHost) != cudaSuccess)
    return DSA_ERR_CUDA;
  return DSA_OK;
}

int dsa_workspace_size(const dsa_problem* p, int32_t algo, const dsa_route_params* rp,
                       size_t* bytes) {
  if (!bytes) return DSA_ERR_INVALID;
  int v = validate_problem(p);
  if (v != DSA_OK) return v;
  if (algo == DSA_ALGO_DSA) {
    *bytes = dsa_layout(p).total;
    return DSA_OK;
  }
  RouteCfg c;
  v = route_cfg(p, algo, rp, &c);
  if (v != DSA_OK) return v;
  *bytes = route_layout(p, c).total;
  return DSA_OK;
}

int dsa_route_chunk_rows(const dsa_problem* p, int32_t algo, const dsa_route_params* rp,
                         int32_t* rows) {
  if (!rows) return DSA_ERR_INVALID;
  int v = validate_problem(p);
  if (v != DSA_OK) return v;
  RouteCfg c;
  v = route_cfg(p, algo, rp, &c);
  if (v != DSA_OK) return v;
  *rows = route_layout(p, c).nq_c;
  return DSA_OK;
}

// DoSA: per-block key ranges into the workspace, then the per-(row, block)
// upper bounds of I into ub [batch * n_q, L.dosa_nblk].
static int run_dosa_bounds(const dsa_problem* p, const DsaLayout& L, const void* q, const void* k,
                    const float* w, uint8_t* ws, float* ub, float* lb, cudaStream_t st) {
  uint16_t* E = reinterpret_cast<uint16_t*>(ws + L.off_ranges);
  float* mx = reinterpret_cast<float*>(ws + L.off_mx);
  dosa_ranges_kernel<<<dim3((unsigned)L.dosa_nblk, (unsigned)p->batch), 128, 0, st>>>(
      reinterpret_cast<const uint16_t*>(k), p->n_k, kDosaShift, L.dosa_nblk, E, mx);
  CUtensorMap qbm, em;
  if (!make_map(&qbm, q, 2, (uint64_t)p->batch * p->n_q * p->heads, 128)) return DSA_ERR_CUDA;
  if (!make_map_ranges(&em, E, (uint64_t)L.dosa_nblk, (uint64_t)p->batch)) return DSA_ERR_CUDA;
  DosaArgs da{};
  da.batch = p->batch;
  da.n_q = p->n_q;
  da.n_tok = p->n_k;
  da.H = p->heads;
  da.shift = kDosaShift;
  da.nblk = L.dosa_nblk;
  da.q_pos0 = p->q_pos0;
  da.k_len = p->k_len;
  da.w = w;
  da.mx = mx;
  da.ub = ub;
  da.lb = lb ? lb : reinterpret_cast<float*>(ws + L.off_lb);
  da.status = reinterpret_cast<int32_t*>(ws);
  if (cudaFuncSetAttribute(dosa_bound_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)dosa_smem_bytes()) != cudaSuccess)
    return DSA_ERR_CUDA;
  const int rpc = 128 / p->heads;
  const int64_t nct = (int64_t)p->batch * ((p->n_q + rpc - 1) / rpc);
  dosa_bound_kernel<<<(unsigned)nct, kDosaThreads, dosa_smem_bytes(), st>>>(qbm, em, da);
  // the seed set: a lower bound of each row's keep-th best score
  const int64_t rows = (int64_t)p->batch * p->n_q;
  dosa_seed_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(
      p->batch, p->n_q, p->n_k, L.dosa_nblk, kDosaShift, p->topk, p->q_pos0, p->k_len, da.lb,
      ub, reinterpret_cast<float*>(ws + L.off_seed),
      reinterpret_cast<unsigned long long*>(ws + offsetof(WsHeader, dosa_blocks)));
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

int dsa_dosa_bounds(const dsa_problem* p, const void* q, const void* k, const float* w,
                    float* ub, float* lb, void* workspace, size_t workspace_bytes, void* stream) {
  int v = validate_problem(p);
  if (v != DSA_OK) return v;
  if (!(p->flags & DSA_FLAG_DOSA)) return DSA_ERR_INVALID;
  if (!q || !k || !w || !ub) return DSA_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k)) return DSA_ERR_INVALID;
  const DsaLayout L = dsa_layout(p);
  if (!workspace || workspace_bytes < L.total) return DSA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return DSA_ERR_INVALID;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  if (cudaMemsetAsync(ws, 0, kWsHeaderBytes, st) != cudaSuccess) return DSA_ERR_CUDA;
  v = run_dosa_bounds(p, L, q, k, w, ws, ub, lb, st);
  if (v != DSA_OK) return v;
  if (p->flags & DSA_FLAG_CHECK) return dsa_read_status(workspace, stream);
  return DSA_OK;
}

int dsa_index_scan(const dsa_problem* p, const void* q, const float* q_scale, const void* k,
                   const float* k_scale, const float* w, void* workspace, size_t workspace_bytes,
                   void* stream) {
  int v = validate_problem(p);
  if (v != DSA_OK) return v;
  if (!q || !k || !w) return DSA_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k)) return DSA_ERR_INVALID;
  if (p->q_dtype == DSA_E4M3 && !q_scale) return DSA_ERR_INVALID;
  if (p->k_dtype == DSA_E4M3 && !k_scale) return DSA_ERR_INVALID;
  const DsaLayout L = dsa_layout(p);
  if (!workspace || workspace_bytes < L.total) return DSA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return DSA_ERR_INVALID;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  int32_t* status = reinterpret_cast<int32_t*>(ws);
  if (cudaMemsetAsync(ws, 0, kWsHeaderBytes, st) != cudaSuccess) return DSA_ERR_CUDA;
  const ScanPlan& pl = L.pl;
  if (p->flags & DSA_FLAG_CHECK) {
    check_inputs_kernel<<<64, 256, 0, st>>>(
        p->q_dtype == DSA_E4M3 ? q_scale : nullptr,
        p->q_dtype == DSA_E4M3 ? (int64_t)p->batch * p->n_q : 0,
        p->k_dtype == DSA_E4M3 ? k_scale : nullptr,
        p->k_dtype == DSA_E4M3 ? (int64_t)p->batch * p->n_k : 0, p->q_pos0, p->k_len, p->batch,
        p->n_k, status);
  }
  const void* qop = q;
  const float* hscale = nullptr;
  if (pl.split) {
    uint8_t* parts = ws + L.off_parts;
    float* hs = reinterpret_cast<float*>(ws + L.off_hscale);
    const int64_t rh = (int64_t)pl.rows * p->heads;
    split_query_kernel<<<(unsigned)((rh + 7) / 8), 256, 0, st>>>(q, p->q_dtype, pl.rows, p->heads,
                                                               p->dim, parts, hs);
    qop = parts;
    hscale = hs;
  }
  CUtensorMap qm, km;
  const int qesz = pl.split ? 1 : pl.esz;
  if (!make_map(&qm, qop, qesz, (uint64_t)pl.rows * p->heads * pl.parts,
                (uint32_t)(pl.qcols / pl.parts)))
    return DSA_ERR_CUDA;
  if (!make_map(&km, k, pl.esz, (uint64_t)p->batch * p->n_k, 128)) return DSA_ERR_CUDA;
  ScanArgs a{};
  a.batch = p->batch;
  a.n_q = p->n_q;
  a.n_k = p->n_k;
  a.H = p->heads;
  a.d = p->dim;
  a.q_stride = p->n_q;
  a.q_off = 0;
  a.n_tok = p->n_k;
  a.bs_shift = 0;
  a.klist = nullptr;
  a.klist_len = 0;
  a.lb_shift = 0;
  a.keep = p->topk;
  a.QG = pl.QG;
  a.qcols = pl.qcols;
  a.kstages = pl.kstages;
  a.kt = pl.kt;
  a.tstages = pl.tstages;
  a.G = pl.G;
  a.stage_cols = pl.stage_cols;
  a.n_qt = pl.n_qt;
  a.C = pl.C;
  a.chunk = pl.chunk;
  a.n_items = pl.n_items;
  a.q_pos0 = p->q_pos0;
  a.k_len = p->k_len;
  a.w = w;
  a.row_scale = p->q_dtype == DSA_E4M3 ? q_scale : nullptr;
  a.head_scale = hscale;
  a.k_scale = p->k_dtype == DSA_E4M3 ? k_scale : nullptr;
  a.nsub = pl.nsub;
  a.capw = pl.capw;
  a.logs = reinterpret_cast<uint64_t*>(ws + L.off_logs);
  a.log_cnt = reinterpret_cast<int32_t*>(ws + L.off_cnt);
  a.log_thr = reinterpret_cast<unsigned long long*>(ws + L.off_thr);
  a.status = status;
  const bool stall = (p->flags & DSA_FLAG_TEST_STALL) != 0;
  a.wait_cycles = stall ? kTestWaitCycles : kWaitCycles;
  a.test_stall = stall ? 1 : 0;
  if (p->flags & DSA_FLAG_DOSA) {
    float* ub = reinterpret_cast<float*>(ws + L.off_ub);
    v = run_dosa_bounds(p, L, q, k, w, ws, ub, nullptr, st);
    if (v != DSA_OK) return v;
    a.dosa_ub = ub;
    a.dosa_seed = reinterpret_cast<const float*>(ws + L.off_seed);
    a.dosa_counts = reinterpret_cast<const unsigned long long*>(ws + offsetof(WsHeader, dosa_blocks));
    a.dosa_nblk = L.dosa_nblk;
    a.dosa_shift = kDosaShift;
    a.dosa_pruned = reinterpret_cast<unsigned long long*>(ws + offsetof(WsHeader, pruned));
  }
  if (launch_scan(pl, qm, km, a, st) != cudaSuccess) return DSA_ERR_CUDA;
  return DSA_OK;
}

int dsa_index_select(const dsa_problem* p, int32_t* out_idx, float* out_score, void* workspace,
                     size_t workspace_bytes, void* stream) {
  int v = validate_problem(p);
  if (v != DSA_OK) return v;
  if (!out_idx || !out_score) return DSA_ERR_INVALID;
  const DsaLayout L = dsa_layout(p);
  if (!workspace || workspace_bytes < L.total) return DSA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return DSA_ERR_INVALID;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  const ScanPlan& pl = L.pl;
  const int sorted = out_order(p);
  if (launch_finalize(pl, p->topk, sorted, reinterpret_cast<const uint64_t*>(ws + L.off_logs),
                      reinterpret_cast<const int32_t*>(ws + L.off_cnt),
                      reinterpret_cast<const unsigned long long*>(ws + L.off_thr), out_idx,
                      out_score, OutMap{p->n_q, p->n_q, 0}, reinterpret_cast<const int32_t*>(ws),
                      st) != cudaSuccess)
    return DSA_ERR_CUDA;
  return finish(p, workspace, st);
}

int dsa_index(const dsa_problem* p, const void* q, const float* q_scale, const void* k,
              const float* k_scale, const float* w, int32_t* out_idx, float* out_score,
              void* workspace, size_t workspace_bytes, void* stream) {
  if (p && (!out_idx || !out_score)) return DSA_ERR_INVALID;
  int rc = dsa_index_scan(p, q, q_scale, k, k_scale, w, workspace, workspace_bytes, stream);
  if (rc != DSA_OK) return rc;
  return dsa_index_select(p, out_idx, out_score, workspace, workspace_bytes, stream);
}

int dsa_index_noalloc(const dsa_problem* p, const void* q, const float* q_scale, const void* k,
                      const float* k_scale, const float* w, int32_t* out_idx, float* out_score,
                      void* stream) {
  int v = validate_problem(p);
  if (v != DSA_OK) return v;
  if (dsa_layout(p).total > kNoAllocScratchBytes) return DSA_ERR_WORKSPACE;
  void* scratch = nullptr;
  const int rc = noalloc_scratch_address(&scratch);
  if (rc != DSA_OK) return rc;
  return dsa_index(p, q, q_scale, k, k_scale, w, out_idx, out_score, scratch,
                   kNoAllocScratchBytes, stream);
}

// ------------------------------------------------------- host-buffer path --
// dsa_index with q, w (and q_scale) in page-locked host memory and the results
// written back to host memory.  The rows stream in chunks through two device
// slots: host->device copies on one internal stream, the scan and select on
// the caller's stream, device->host copies on another, so the copies of one
// chunk overlap the scan of its neighbours.  Staging layout: a 256-byte header
// (the call's status, first error over all chunks), then per slot q, w,
// q_scale, the chunk's causal offsets and its results, then the workspace of
// one chunk.

}  // extern "C"

namespace {

__global__ void chunk_meta_kernel(const int32_t* q_pos0, const int32_t* k_len, int b, int r0,
                                  int n_q, int n_k, int32_t* meta) {
  meta[0] = (q_pos0 ? q_pos0[b] : n_k - n_q) + r0;
  meta[1] = k_len ? k_len[b] : n_k;
}

__global__ void sticky_status_kernel(const int32_t* chunk_status, int32_t* call_status) {
  if (call_status[0] == DSA_OK && chunk_status[0] != DSA_OK) {
    call_status[0] = chunk_status[0];
    call_status[1] = chunk_status[1];
  }
}

struct HostLayout {
  int rows;                      // rows per chunk
  size_t q_row, w_row;           // bytes per query row
  size_t off_q[2], off_w[2], off_qs[2], off_meta[2], off_idx[2], off_sc[2], off_ws;
  size_t ws_bytes, total;
};

int host_layout(const dsa_problem* p, int chunk_rows, HostLayout* L) {
  if (chunk_rows < 1) return DSA_ERR_INVALID;
  L->rows = std::min(chunk_rows, p->n_q);
  const int qesz = p->q_dtype == DSA_F32 ? 4 : (p->q_dtype == DSA_BF16 ? 2 : 1);
  L->q_row = (size_t)p->heads * p->dim * qesz;
  L->w_row = (size_t)p->heads * sizeof(float);
  dsa_problem c = *p;
  c.batch = 1;
  c.n_q = L->rows;
  const size_t R = (size_t)L->rows;
  size_t off = kWsHeaderBytes;
  for (int s = 0; s < 2; ++s) {
    L->off_q[s] = off;
    off += align_up(R * L->q_row);
    L->off_w[s] = off;
    off += align_up(R * L->w_row);
    L->off_qs[s] = off;
    if (p->q_dtype == DSA_E4M3) off += align_up(R * sizeof(float));
    L->off_meta[s] = off;
    off += align_up(2 * sizeof(int32_t));
    L->off_idx[s] = off;
    off += align_up(R * p->topk * sizeof(int32_t));
    L->off_sc[s] = off;
    off += align_up(R * p->topk * sizeof(float));
  }
  L->off_ws = off;
  L->ws_bytes = dsa_layout(&c).total;
  L->total = off + align_up(L->ws_bytes);
  return DSA_OK;
}

constexpr int kHostMaxDevices = 64;
std::mutex g_host_mu;
cudaStream_t g_host_h2d[kHostMaxDevices], g_host_d2h[kHostMaxDevices];

// The two copy streams of the current device, created once (non-blocking).
int host_streams(cudaStream_t* h2d, cudaStream_t* d2h) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kHostMaxDevices) {
    cudaGetLastError();
    return DSA_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_host_mu);
  if (!g_host_h2d[dev]) {
    if (cudaStreamCreateWithFlags(&g_host_h2d[dev], cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&g_host_d2h[dev], cudaStreamNonBlocking) != cudaSuccess) {
      cudaGetLastError();
      return DSA_ERR_CUDA;
    }
  }
  *h2d = g_host_h2d[dev];
  *d2h = g_host_d2h[dev];
  return DSA_OK;
}

}  // namespace

extern "C" {

int dsa_host_staging_size(const dsa_problem* p, int32_t chunk_rows, size_t* bytes) {
  if (!bytes) return DSA_ERR_INVALID;
  int v = validate_problem(p);
  if (v != DSA_OK) return v;
  HostLayout L;
  v = host_layout(p, chunk_rows, &L);
  if (v != DSA_OK) return v;
  *bytes = L.total;
  return DSA_OK;
}

int dsa_index_host(const dsa_problem* p, const void* q_host, const float* q_scale_host,
                   const void* k, const float* k_scale, const float* w_host,
                   int32_t* idx_host, float* score_host, int32_t chunk_rows, void* staging,
                   size_t staging_bytes, void* stream) {
  int v = validate_problem(p);
  if (v != DSA_OK) return v;
  if (!q_host || !k || !w_host || !idx_host || !score_host) return DSA_ERR_INVALID;
  if (p->q_dtype == DSA_E4M3 && !q_scale_host) return DSA_ERR_INVALID;
  if (p->k_dtype == DSA_E4M3 && !k_scale) return DSA_ERR_INVALID;
  if (!aligned16(k)) return DSA_ERR_INVALID;
  HostLayout L;
  v = host_layout(p, chunk_rows, &L);
  if (v != DSA_OK) return v;
  if (!staging || staging_bytes < L.total) return DSA_ERR_WORKSPACE;
  if (!aligned16(staging)) return DSA_ERR_INVALID;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream), h2d, d2h;
  v = host_streams(&h2d, &d2h);
  if (v != DSA_OK) return v;
  uint8_t* sg = reinterpret_cast<uint8_t*>(staging);
  int32_t* call_status = reinterpret_cast<int32_t*>(sg);
  void* ws = sg + L.off_ws;
  const int kesz = p->k_dtype == DSA_F32 ? 4 : (p->k_dtype == DSA_BF16 ? 2 : 1);
  const size_t k_seq = (size_t)p->n_k * p->dim * kesz;
  cudaEvent_t start, h2d_done[2], comp_done[2], d2h_done[2];
  cudaEvent_t* evs[7] = {&start, &h2d_done[0], &h2d_done[1], &comp_done[0], &comp_done[1],
                         &d2h_done[0], &d2h_done[1]};
  int made = 0;
  for (; made < 7; ++made)
    if (cudaEventCreateWithFlags(evs[made], cudaEventDisableTiming) != cudaSuccess) break;
  int rc = made == 7 ? DSA_OK : DSA_ERR_CUDA;
  int c = 0;
  if (rc == DSA_OK) {
    // the copy streams start after the caller's earlier work on its stream
    if (cudaMemsetAsync(sg, 0, kWsHeaderBytes, st) != cudaSuccess ||
        cudaEventRecord(start, st) != cudaSuccess || cudaStreamWaitEvent(h2d, start, 0) != cudaSuccess ||
        cudaStreamWaitEvent(d2h, start, 0) != cudaSuccess)
      rc = DSA_ERR_CUDA;
  }
  for (int b = 0; b < p->batch && rc == DSA_OK; ++b) {
    for (int r0 = 0; r0 < p->n_q && rc == DSA_OK; r0 += L.rows, ++c) {
      const int n = std::min(L.rows, p->n_q - r0);
      const int s = c & 1;
      const size_t row0 = (size_t)b * p->n_q + r0;
      bool ok = true;
      // slot s: its inputs free once chunk c - 2 was scanned, its results once copied out
      if (c >= 2) ok = ok && cudaStreamWaitEvent(h2d, comp_done[s], 0) == cudaSuccess;
      ok = ok && cudaMemcpyAsync(sg + L.off_q[s], reinterpret_cast<const uint8_t*>(q_host) + row0 * L.q_row,
                                 (size_t)n * L.q_row, cudaMemcpyHostToDevice, h2d) == cudaSuccess;
      ok = ok && cudaMemcpyAsync(sg + L.off_w[s], w_host + row0 * p->heads, (size_t)n * L.w_row,
                                 cudaMemcpyHostToDevice, h2d) == cudaSuccess;
      if (p->q_dtype == DSA_E4M3)
        ok = ok && cudaMemcpyAsync(sg + L.off_qs[s], q_scale_host + row0, (size_t)n * sizeof(float),
                                   cudaMemcpyHostToDevice, h2d) == cudaSuccess;
      ok = ok && cudaEventRecord(h2d_done[s], h2d) == cudaSuccess;
      ok = ok && cudaStreamWaitEvent(st, h2d_done[s], 0) == cudaSuccess;
      if (c >= 2) ok = ok && cudaStreamWaitEvent(st, d2h_done[s], 0) == cudaSuccess;
      if (!ok) {
        rc = DSA_ERR_CUDA;
        break;
      }
      int32_t* meta = reinterpret_cast<int32_t*>(sg + L.off_meta[s]);
      chunk_meta_kernel<<<1, 1, 0, st>>>(p->q_pos0, p->k_len, b, r0, p->n_q, p->n_k, meta);
      dsa_problem cp = *p;
      cp.batch = 1;
      cp.n_q = n;
      cp.q_pos0 = meta;
      cp.k_len = meta + 1;
      cp.flags = p->flags & ~DSA_FLAG_CHECK;
      int32_t* idx_d = reinterpret_cast<int32_t*>(sg + L.off_idx[s]);
      float* sc_d = reinterpret_cast<float*>(sg + L.off_sc[s]);
      rc = dsa_index(&cp, sg + L.off_q[s],
                     p->q_dtype == DSA_E4M3 ? reinterpret_cast<const float*>(sg + L.off_qs[s]) : nullptr,
                     reinterpret_cast<const uint8_t*>(k) + (size_t)b * k_seq,
                     k_scale ? k_scale + (size_t)b * p->n_k : nullptr,
                     reinterpret_cast<const float*>(sg + L.off_w[s]), idx_d, sc_d, ws, L.ws_bytes, st);
      if (rc != DSA_OK) break;
      sticky_status_kernel<<<1, 1, 0, st>>>(reinterpret_cast<const int32_t*>(ws), call_status);
      ok = cudaEventRecord(comp_done[s], st) == cudaSuccess &&
           cudaStreamWaitEvent(d2h, comp_done[s], 0) == cudaSuccess &&
           cudaMemcpyAsync(idx_host + row0 * p->topk, idx_d, (size_t)n * p->topk * sizeof(int32_t),
                           cudaMemcpyDeviceToHost, d2h) == cudaSuccess &&
           cudaMemcpyAsync(score_host + row0 * p->topk, sc_d, (size_t)n * p->topk * sizeof(float),
                           cudaMemcpyDeviceToHost, d2h) == cudaSuccess &&
           cudaEventRecord(d2h_done[s], d2h) == cudaSuccess;
      if (!ok) rc = DSA_ERR_CUDA;
    }
  }
  // the caller's stream continues once every result has reached the host
  if (rc == DSA_OK) {
    for (int s = 0; s < 2 && s < c; ++s)
      if (cudaStreamWaitEvent(st, d2h_done[s], 0) != cudaSuccess) rc = DSA_ERR_CUDA;
  }
  for (int i = 0; i < made; ++i) cudaEventDestroy(*evs[i]);
  if (rc != DSA_OK) {
    cudaGetLastError();
    return rc;
  }
  if (cudaPeekAtLastError() != cudaSuccess) {
    cudaGetLastError();
    return DSA_ERR_CUDA;
  }
  if (p->flags & DSA_FLAG_CHECK) return dsa_read_status(staging, stream);
  return DSA_OK;
}

int dsa_quantize_e4m3(const void* x, int32_t x_dtype, int64_t rows, int32_t cols, uint8_t* out,
                      float* out_scale, void* stream) {
  if (!x || !out || !out_scale || rows < 0 || cols < 1) return DSA_ERR_INVALID;
  if (x_dtype != DSA_F32 && x_dtype != DSA_BF16) return DSA_ERR_UNSUPPORTED;
  if (rows == 0) return DSA_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  quantize_rows_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(x, x_dtype, rows, cols, out,
                                                                   out_scale);
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

int misa_index(const dsa_problem* p, const dsa_route_params* rp, const void* q, const void* k,
               const float* w, int32_t* out_idx, float* out_score, int32_t* out_heads,
               float* out_E, void* workspace, size_t workspace_bytes, void* stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  RouteLayout L;
  int rc = route_begin(p, DSA_ALGO_MISA, rp, q, k, w, out_idx, out_score, workspace,
                       workspace_bytes, st, &L);
  if (rc != DSA_OK) return rc;
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  int32_t* status = reinterpret_cast<int32_t*>(ws);
  int32_t* heads = out_heads ? out_heads : reinterpret_cast<int32_t*>(ws + L.off_heads);
  rc = run_router(p, L, q, k, w, heads, out_E, ws, st);
  if (rc != DSA_OK) return rc;
  const int sorted = out_order(p);
  for (int ci = 0; ci < L.n_chunks; ++ci) {
    const int q_off = ci * L.nq_c;
    const int nq = p->n_q - q_off < L.nq_c ? p->n_q - q_off : L.nq_c;
    const RouteStages rs = plan_route(p, L.c, nq);
    const LogPtrs lp = log_ptrs(rs.s1, ws + L.off_logs);
    StageIO io{};
    io.q = ws + L.off_qg;
    io.w = reinterpret_cast<const float*>(ws + L.off_wg);
    io.q_stride = p->n_q;
    io.H = L.c.h;
    io.k = k;
    io.k_rows = (uint64_t)p->batch * p->n_k;
    io.k_box = 128;
    io.n_kmap = p->n_k;
    rc = run_stage(p, rs.s1, io, q_off, nq, lp, status, st);
    if (rc != DSA_OK) return rc;
    if (launch_finalize(rs.s1, p->topk, sorted, lp.logs, lp.cnt, lp.thr, out_idx, out_score,
                        OutMap{nq, p->n_q, q_off}, status, st) != cudaSuccess)
      return DSA_ERR_CUDA;
  }
  return finish(p, workspace, st);
}

int misa_dagger_index(const dsa_problem* p, const dsa_route_params* rp, const void* q,
                      const void* k, const float* w, int32_t* out_idx, float* out_score,
                      int32_t* out_heads, int32_t* out_pool, void* workspace,
                      size_t workspace_bytes, void* stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  RouteLayout L;
  int rc = route_begin(p, DSA_ALGO_MISA_DAGGER, rp, q, k, w, out_idx, out_score, workspace,
                       workspace_bytes, st, &L);
  if (rc != DSA_OK) return rc;
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  int32_t* status = reinterpret_cast<int32_t*>(ws);
  int32_t* heads = out_heads ? out_heads : reinterpret_cast<int32_t*>(ws + L.off_heads);
  rc = run_router(p, L, q, k, w, heads, nullptr, ws, st);
  if (rc != DSA_OK) return rc;
  const int sorted = out_order(p);
  int32_t* pool = reinterpret_cast<int32_t*>(ws + L.off_list);
  for (int ci = 0; ci < L.n_chunks; ++ci) {
    const int q_off = ci * L.nq_c;
    const int nq = p->n_q - q_off < L.nq_c ? p->n_q - q_off : L.nq_c;
    const RouteStages rs = plan_route(p, L.c, nq);
    // pass 1: routed heads, keep k' candidates
    LogPtrs lp = log_ptrs(rs.s1, ws + L.off_logs);
    StageIO io{};
    io.q = ws + L.off_qg;
    io.w = reinterpret_cast<const float*>(ws + L.off_wg);
    io.q_stride = p->n_q;
    io.H = L.c.h;
    io.k = k;
    io.k_rows = (uint64_t)p->batch * p->n_k;
    io.k_box = 128;
    io.n_kmap = p->n_k;
    rc = run_stage(p, rs.s1, io, q_off, nq, lp, status, st);
    if (rc != DSA_OK) return rc;
    if (launch_finalize(rs.s1, L.c.kp, 0, lp.logs, lp.cnt, lp.thr, pool, nullptr,
                        OutMap{nq, nq, 0}, status, st) != cudaSuccess)
      return DSA_ERR_CUDA;
    if (out_pool) {
      rc = copy_lists(out_pool, pool, p, q_off, nq, L.c.kp, st);
      if (rc != DSA_OK) return rc;
    }
    // pass 2: every head on the pool's tokens
    lp = log_ptrs(rs.s2, ws + L.off_logs);
    StageIO io2{};
    io2.q = q;
    io2.w = w;
    io2.q_stride = p->n_q;
    io2.H = p->heads;
    io2.k = k;
    io2.k_rows = (uint64_t)p->batch * p->n_k;
    io2.k_box = 1;                      // gather4 rows
    io2.n_kmap = p->n_k;
    io2.klist = pool;
    io2.klist_len = L.c.kp;
    io2.gather = 1;
    rc = run_stage(p, rs.s2, io2, q_off, nq, lp, status, st);
    if (rc != DSA_OK) return rc;
    if (launch_finalize(rs.s2, p->topk, sorted, lp.logs, lp.cnt, lp.thr, out_idx, out_score,
                        OutMap{nq, p->n_q, q_off}, status, st) != cudaSuccess)
      return DSA_ERR_CUDA;
  }
  return finish(p, workspace, st);
}

int hisa_index(const dsa_problem* p, const dsa_route_params* rp, const void* q, const void* k,
               const float* w, int32_t* out_idx, float* out_score, int32_t* out_blocks,
               int32_t* out_heads, void* workspace, size_t workspace_bytes, void* stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  RouteLayout L;
  int rc = route_begin(p, DSA_ALGO_HISA, rp, q, k, w, out_idx, out_score, workspace,
                       workspace_bytes, st, &L);
  if (rc != DSA_OK) return rc;
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  int32_t* status = reinterpret_cast<int32_t*>(ws);
  const RouteCfg& c = L.c;
  const void* qs = q;
  const float* wsrc = w;
  if (c.route) {
    int32_t* heads = out_heads ? out_heads : reinterpret_cast<int32_t*>(ws + L.off_heads);
    rc = run_router(p, L, q, k, w, heads, nullptr, ws, st);
    if (rc != DSA_OK) return rc;
    qs = ws + L.off_qg;
    wsrc = reinterpret_cast<const float*>(ws + L.off_wg);
  }
  uint8_t* runH = ws + L.off_runH;
  uint8_t* fullH = ws + L.off_fullH;
  rc = launch_pool(k, p, c.bsH, runH, fullH, c.nblkH, st);
  if (rc != DSA_OK) return rc;
  const int sorted = out_order(p);
  int32_t* blocks = reinterpret_cast<int32_t*>(ws + L.off_list);
  for (int ci = 0; ci < L.n_chunks; ++ci) {
    const int q_off = ci * L.nq_c;
    const int nq = p->n_q - q_off < L.nq_c ? p->n_q - q_off : L.nq_c;
    const RouteStages rs = plan_route(p, c, nq);
    // coarse: the full blocks' representatives scored like keys, keep r
    LogPtrs lp = log_ptrs(rs.s1, ws + L.off_logs);
    StageIO io{};
    io.q = qs;
    io.w = wsrc;
    io.q_stride = p->n_q;
    io.H = c.hh;
    io.k = fullH;
    io.k_rows = L.fullH_rows;
    io.k_box = 128;
    io.n_kmap = c.nblkH > 0 ? c.nblkH : 1;
    io.bs_shift = c.bsH;
    rc = run_stage(p, rs.s1, io, q_off, nq, lp, status, st);
    if (rc != DSA_OK) return rc;
    // the boundary block of every row joins its candidates
    BoundaryArgs ba{};
    ba.batch = p->batch;
    ba.n_q = nq;
    ba.q_stride = p->n_q;
    ba.q_off = q_off;
    ba.n_tok = p->n_k;
    ba.H = c.hh;
    ba.bs_shift = c.bsH;
    ba.q_pos0 = p->q_pos0;
    ba.k_len = p->k_len;
    ba.q = reinterpret_cast<const uint16_t*>(qs);
    ba.w = wsrc;
    ba.run = reinterpret_cast<const uint16_t*>(runH);
    ba.C = rs.s1.C;
    ba.nsub = rs.s1.nsub;
    ba.capw = rs.s1.capw;
    ba.logs = lp.logs;
    ba.log_cnt = lp.cnt;
    const long long rows = (long long)p->batch * nq;
    boundary_candidate_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(ba);
    if (cudaGetLastError() != cudaSuccess) return DSA_ERR_CUDA;
    if (launch_finalize(rs.s1, c.r, 0, lp.logs, lp.cnt, lp.thr, blocks, nullptr,
                        OutMap{nq, nq, 0}, status, st) != cudaSuccess)
      return DSA_ERR_CUDA;
    if (out_blocks) {
      rc = copy_lists(out_blocks, blocks, p, q_off, nq, c.r, st);
      if (rc != DSA_OK) return rc;
    }
    // fine: the kept blocks' legal tokens with the full formula
    lp = log_ptrs(rs.s2, ws + L.off_logs);
    StageIO io2{};
    io2.q = qs;
    io2.w = wsrc;
    io2.q_stride = p->n_q;
    io2.H = c.hh;
    io2.k = k;
    io2.k_rows = (uint64_t)p->batch * p->n_k;
    io2.k_box = c.bsH < 7 ? (1u << c.bsH) : 128u;
    io2.n_kmap = p->n_k;
    io2.klist = blocks;
    io2.klist_len = c.r;
    io2.lb_shift = c.bsH;
    io2.gather = 2;
    rc = run_stage(p, rs.s2, io2, q_off, nq, lp, status, st);
    if (rc != DSA_OK) return rc;
    if (launch_finalize(rs.s2, p->topk, sorted, lp.logs, lp.cnt, lp.thr, out_idx, out_score,
                        OutMap{nq, p->n_q, q_off}, status, st) != cudaSuccess)
      return DSA_ERR_CUDA;
  }
  return finish(p, workspace, st);
}

int lisa_index(const dsa_problem* p, const dsa_route_params* rp, const void* q, const void* k,
               const float* w, int32_t* out_idx, float* out_score, int32_t* out_pool,
               void* workspace, size_t workspace_bytes, void* stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  RouteLayout L;
  int rc = route_begin(p, DSA_ALGO_LISA, rp, q, k, w, out_idx, out_score, workspace,
                       workspace_bytes, st, &L);
  if (rc != DSA_OK) return rc;
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  rc = run_pseudo(p, L, q, w, nullptr, ws, st);
  if (rc != DSA_OK) return rc;
  rc = run_pseudo_stages(p, L, q, k, w, out_idx, out_score, out_pool, ws, st);
  if (rc != DSA_OK) return rc;
  return finish(p, workspace, st);
}

int resmisa_index(const dsa_problem* p, const dsa_route_params* rp, const void* q, const void* k,
                  const float* w, int32_t* out_idx, float* out_score, int32_t* out_heads,
                  float* out_S, void* workspace, size_t workspace_bytes, void* stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  RouteLayout L;
  int rc = route_begin(p, DSA_ALGO_RESMISA, rp, q, k, w, out_idx, out_score, workspace,
                       workspace_bytes, st, &L);
  if (rc != DSA_OK) return rc;
  uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
  const RouteCfg& c = L.c;
  int32_t* heads = out_heads ? out_heads : reinterpret_cast<int32_t*>(ws + L.off_heads);
  uint16_t* ext_run = reinterpret_cast<uint16_t*>(ws + L.off_extrun);
  uint16_t* ext_full = reinterpret_cast<uint16_t*>(ws + L.off_extfull);
  if (c.res_r > 0) {
    const int nb = (p->n_k + (1 << c.bsX) - 1) >> c.bsX;
    block_extrema_kernel<<<dim3((unsigned)nb, (unsigned)p->batch), 128, 0, st>>>(
        reinterpret_cast<const uint16_t*>(k), p->n_k, c.bsX, ext_run, ext_full, c.nblkX);
    if (cudaGetLastError() != cudaSuccess) return DSA_ERR_CUDA;
    ResRouterArgs ra{};
    ra.batch = p->batch;
    ra.n_q = p->n_q;
    ra.n_tok = p->n_k;
    ra.H = p->heads;
    ra.r = c.res_r;
    ra.bs_shift = c.bsX;
    ra.nblk_full = c.nblkX;
    ra.q_pos0 = p->q_pos0;
    ra.k_len = p->k_len;
    ra.q = reinterpret_cast<const uint16_t*>(q);
    ra.w = w;
    ra.ext_full = ext_full;
    ra.ext_run = ext_run;
    ra.heads = heads;
    ra.S = out_S;
    const int rpc = kResThreads / p->heads;
    const long long ctas = (long long)p->batch * ((p->n_q + rpc - 1) / rpc);
    residual_router_kernel<<<(unsigned)ctas, kResThreads, 0, st>>>(ra);
    if (cudaGetLastError() != cudaSuccess) return DSA_ERR_CUDA;
  }
  rc = run_pseudo(p, L, q, w, heads, ws, st);
  if (rc != DSA_OK) return rc;
  rc = run_pseudo_stages(p, L, q, k, w, out_idx, out_score, nullptr, ws, st);
  if (rc != DSA_OK) return rc;
  return finish(p, workspace, st);
}

int dsa_sparse_mla(const dsa_mla_problem* p, const void* q, const void* kv, const int32_t* idx,
                   void* out, float* out_lse, void* workspace, size_t workspace_bytes,
                   void* stream) {
  if (!p || !q || !kv || !idx || !out) return DSA_ERR_INVALID;
  if (p->batch < 1 || p->tokens_per_seq < 1 || p->n_k < 1 || p->heads < 1 || p->topk < 1)
    return DSA_ERR_INVALID;
  if (p->dim_qk != kMlaDqk || p->dim_v != kMlaDv || p->heads > 128 || p->topk > 65536)
    return DSA_ERR_UNSUPPORTED;
  const long long T = (long long)p->batch * p->tokens_per_seq;
  if (T * 2 > 0x7fffffffll || (long long)p->batch * p->n_k > (1ll << 31)) return DSA_ERR_UNSUPPORTED;
  if (!(p->scale > 0.f) || !(p->scale < 3.0e38f)) return DSA_ERR_INVALID;
  if (!aligned16(q) || !aligned16(kv) || !aligned16(out) || !aligned16(idx))
    return DSA_ERR_INVALID;
  if (!workspace || workspace_bytes < kWsHeaderBytes) return DSA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return DSA_ERR_INVALID;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int32_t* status = reinterpret_cast<int32_t*>(workspace);
  if (cudaMemsetAsync(workspace, 0, kWsHeaderBytes, st) != cudaSuccess) return DSA_ERR_CUDA;
  CUtensorMap qm, km;
  if (!make_map_q3d(&qm, q, (uint64_t)T, (uint64_t)p->heads)) return DSA_ERR_CUDA;
  if (!make_map_kv(&km, kv, (uint64_t)p->batch * p->n_k)) return DSA_ERR_CUDA;
  MlaArgs a{};
  a.T = (int32_t)T;
  a.tps = p->tokens_per_seq;
  a.n_k = p->n_k;
  a.heads = p->heads;
  a.topk = p->topk;
  a.scale_log2 = p->scale * 1.4426950408889634f;
  a.idx = idx;
  a.out = reinterpret_cast<uint16_t*>(out);
  a.lse = out_lse;
  a.status = status;
  const int smem = (int)mla_smem_bytes();
  if (cudaFuncSetAttribute(sparse_mla_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess)
    return DSA_ERR_CUDA;
  sparse_mla_kernel<<<(unsigned)(T * 2), kMlaThreads, smem, st>>>(qm, km, a);
  if (cudaGetLastError() != cudaSuccess) return DSA_ERR_CUDA;
  if (p->flags & DSA_FLAG_CHECK) return dsa_read_status(workspace, stream);
  return DSA_OK;
}

int dsa_indexer_backward(const dsa_problem* p, const void* q, const void* k, const float* w,
                         const int32_t* sel, const float* grad, float* dq, float* dk, float* dw,
                         void* workspace, size_t workspace_bytes, void* stream) {
  if (!p || !q || !k || !w || !sel || !grad || !dq || !dk || !dw) return DSA_ERR_INVALID;
  if (p->batch < 1 || p->n_q < 1 || p->n_k < 1 || p->topk < 1) return DSA_ERR_INVALID;
  if (p->dim != 128 || p->heads != kBwdH || p->q_dtype != DSA_BF16 || p->k_dtype != DSA_BF16)
    return DSA_ERR_UNSUPPORTED;
  const long long rows = (long long)p->batch * p->n_q;
  if (rows > 0x7fffffffll || rows * kBwdH > (1ll << 31) ||
      (long long)p->batch * p->n_k > (1ll << 31) || p->topk > (1 << 20))
    return DSA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(dq) || !aligned16(dk)) return DSA_ERR_INVALID;
  if (!workspace || workspace_bytes < kWsHeaderBytes) return DSA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return DSA_ERR_INVALID;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(workspace, 0, kWsHeaderBytes, st) != cudaSuccess) return DSA_ERR_CUDA;
  CUtensorMap qm, km;
  if (!make_map(&qm, q, 2, (uint64_t)rows * kBwdH, kBwdH)) return DSA_ERR_CUDA;
  if (!make_map(&km, k, 2, (uint64_t)p->batch * p->n_k, 1)) return DSA_ERR_CUDA;
  BwdArgs a{};
  a.rows = (int32_t)rows;
  a.n_q = p->n_q;
  a.n_k = p->n_k;
  a.topk = p->topk;
  a.sel = sel;
  a.grad = grad;
  a.w = w;
  a.dq = dq;
  a.dk = dk;
  a.dw = dw;
  a.status = reinterpret_cast<int32_t*>(workspace);
  const int smem = (int)bwd_smem_bytes();
  if (cudaFuncSetAttribute(indexer_backward_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           smem) != cudaSuccess)
    return DSA_ERR_CUDA;
  indexer_backward_kernel<<<(unsigned)rows, kBwdThreads, smem, st>>>(qm, km, a);
  if (cudaGetLastError() != cudaSuccess) return DSA_ERR_CUDA;
  if (p->flags & DSA_FLAG_CHECK) return dsa_read_status(workspace, stream);
  return DSA_OK;
}

}  // extern "C"

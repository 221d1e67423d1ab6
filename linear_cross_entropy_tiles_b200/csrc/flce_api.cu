// flce_api.cu -- C ABI, argument checks, planning and launch sequence of the
// fused linear cross-entropy library.  The operation and every entry point
// are documented in include/flce.h.
//
// Two schedules.  flce_fused on bf16 problems of 512 rows or more runs the
// fused-in-forward schedule (6*BT*H*V FLOP), described above
// enqueue_fused_forward: row chunks whose forward GEMM keeps q = exp(y), then
// dX and dW per chunk.  The forward and backward entry points, fp32 problems
// and small batches run the recompute schedule (two passes over the
// vocabulary, nothing of size BT x V in HBM):
//   forward   labels_kernel -> logit GEMM X W^T with the online-LSE epilogue
//             (per-(tile,row) max / sum-exp partials + target logit)
//             -> combine_kernel (lse, per-row NLL) -> finalize_kernel (loss)
//   backward  labels_kernel, then for each vocabulary chunk [v0, v0+Vc):
//             logit GEMM X W_c^T with the G epilogue -> G_c (bf16, BT x Vc)
//             -> dX (+)= G_c W_c   (fp32 running sum, bf16 on the last chunk)
//             -> dW_c  = G_c^T X   (complete per chunk: its K is all of BT)
// The logits of the backward are recomputed from X, W and the saved lse
// instead of being stored (PyTorch PR #126348, point b: the softmax is rebuilt
// from softmax_input and the small per-row statistics, never saved).
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "flce.h"
#include "internal.h"
#include "aux_kernels.cuh"
#include "gemm_tc.cuh"
#include "gemm_tc2.cuh"
#include "sm100.cuh"

using namespace flce;

namespace {

std::atomic<unsigned long long> g_wait_limit_ns{2000000000ull};
thread_local int32_t t_launches = 0;

// Kernel kinds, in the order flce_kernel_name() names them.
enum Kind : int32_t {
  K_LABELS = 0, K_LSE_GEMM, K_COMBINE, K_FINALIZE, K_GRAD_GEMM, K_DX_GEMM, K_DW_GEMM,
  K_SIMT_LOGITS, K_SIMT_GRAD, K_SIMT_DX, K_SIMT_DW, K_MEMSET, K_LSEQ_GEMM, K_LSEQ,
  K_DWACC_GEMM, K_DX_REDUCE, K_COUNT_VALID, K_SET_NVALID, K_SHIFT_LABELS,
  // launched from flce_ce.cu (kinds fixed in internal.h)
  K_CE_FORWARD, K_CE_BACKWARD, K_CE_FUSED,
  K_LSEQ_REPAIR, K_VP_STATS, K_VP_COMBINE, K_NUM_KINDS
};
static_assert(int32_t(K_CE_FORWARD) == int32_t(flce_internal::kKindCeForward) &&
                  int32_t(K_CE_BACKWARD) == int32_t(flce_internal::kKindCeBackward) &&
                  int32_t(K_CE_FUSED) == int32_t(flce_internal::kKindCeFused),
              "kernel kinds shared with flce_ce.cu");
const char* const kKindNames[K_NUM_KINDS] = {
    "labels", "lse_gemm", "lse_combine", "loss_finalize", "grad_gemm", "dx_gemm", "dw_gemm",
    "simt_lse", "simt_grad", "simt_dx", "simt_dw", "memset", "lse_q_gemm", "lse_q",
    "dw_acc_gemm", "dx_reduce", "count_valid", "set_n_valid", "shift_labels", "ce_forward",
    "ce_backward", "ce_fused", "lse_q_repair_gemm", "vp_stats", "vp_combine"};

// flce_fused schedule: 0 = choose, 1 = two-pass recompute, 2 = fused-in-forward.
std::atomic<int32_t> g_schedule{0};
// Cap on the workspace the automatic schedule may plan (0 = none).
std::atomic<unsigned long long> g_ws_limit{0};

// Optional per-launch CUDA-event timing (flce_profile_start / _stop).
struct Profiler {
  std::mutex mu;
  bool on = false;
  int cap = 0, n = 0;
  cudaEvent_t* ev = nullptr;  // 2 per record: before, after
  int32_t* kind = nullptr;
} g_prof;

void prof_before(cudaStream_t st) {
  if (!g_prof.on || g_prof.n >= g_prof.cap) return;
  cudaEventRecord(g_prof.ev[2 * g_prof.n], st);
}
void prof_after(cudaStream_t st, int32_t kind) {
  ++t_launches;
  if (!g_prof.on || g_prof.n >= g_prof.cap) return;
  cudaEventRecord(g_prof.ev[2 * g_prof.n + 1], st);
  g_prof.kind[g_prof.n++] = kind;
}

constexpr int kStagesBN256 = 4;
constexpr size_t kHeaderBytes = 256;

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }
// Most vocabulary slices dW may be handed over in (flce_fused_global_sliced).
constexpr int32_t kMaxDwSlices = 64;
int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

// ------------------------------- planning ----------------------------------

struct Plan {
  int64_t BT = 0, H = 0, V = 0;
  int64_t ldx = 0, ldw = 0, lddx = 0, lddw = 0;  // row strides (elements) of X, W, dX, dW
  bool dw_f32 = false;    // bf16 inputs with an fp32 dW (the fused schedule sums into dW)
  bool dx_f32 = false;    // bf16 inputs with an fp32 dX (vocabulary-parallel partial sums)
  int64_t label_off = 0;  // vocabulary id of W's first row (vocabulary-parallel slice)
  size_t off_shift = 0;   // shifted labels [BT] int64 when the op shifts token ids
  bool tc = false;        // bf16 tensor-core path (else fp32 SIMT)
  int bn = 256;           // N tile of the logit GEMMs and of dX / dW
  int64_t Vc = 0;         // vocabulary chunk width of the backward
  int64_t n_chunks = 0;
  int64_t ldg = 0;        // row stride of the G chunk buffer, elements
  int64_t part_tiles = 0; // vocabulary slices of the forward partial array
  int part_shift = 8;     // log2 of the columns per partial slice
  size_t g_elem = 2;
  size_t off_lse = 0, off_target = 0, off_rowloss = 0, off_partial = 0, off_g = 0,
         off_dxacc = 0, total = 0;
  // fused-in-forward schedule (flce_fused, bf16): row chunks of Cb rows whose
  // p = exp(y - reference) live in P [Cb][ldp]; dW summed in fp32 over chunks
  bool fused_fwd = false;
  int64_t Cb = 0, n_row_chunks = 0, ldp = 0;
  int dx_splits = 1;      // K (vocabulary) splits of the chunk's dX GEMM
  size_t off_p = 0, off_dwacc = 0, off_dxslab = 0;
  // per chunk row: prescaled X rows [Cb][H] bf16, exponent reference and dX
  // factor; one recomputation flag per 32-row group
  size_t off_xs = 0, off_ref = 0, off_rowscale = 0, off_flags = 0;
};

bool softcap_on(float c) { return c > 0.f && std::isfinite(c); }

flce_status_t check_problem(const flce_problem_t* p) {
  if (!p) return FLCE_ERR_INVALID_ARG;
  if ((p->dw_fp32 != 0 && p->dw_fp32 != 1) || p->shift_seq_len < 0) return FLCE_ERR_INVALID_ARG;
  if (p->shift_seq_len > 0 && p->BT % p->shift_seq_len != 0) return FLCE_ERR_INVALID_ARG;
  if (p->BT < 0 || p->H <= 0 || p->V <= 0) return FLCE_ERR_INVALID_ARG;
  if (p->dtype != FLCE_BF16 && p->dtype != FLCE_FP32) return FLCE_ERR_UNSUPPORTED;
  if (p->H % 8 != 0) return FLCE_ERR_MISALIGNED;
  if (p->BT >= (int64_t(1) << 31) || p->V >= (int64_t(1) << 31) || p->H >= (int64_t(1) << 31))
    return FLCE_ERR_UNSUPPORTED;
  // Row strides: 0 = H; at least H; rows on 16-byte boundaries.
  const int64_t esz = p->dtype == FLCE_BF16 ? 2 : 4;
  const int64_t dw_esz = p->dw_fp32 ? 4 : esz;
  const int64_t lds[4] = {p->ldx, p->ldw, p->lddx, p->lddw};
  for (int i = 0; i < 4; ++i) {
    const int64_t ld = lds[i];
    if (ld < 0 || (ld != 0 && ld < p->H)) return FLCE_ERR_INVALID_ARG;
    if (ld >= (int64_t(1) << 31)) return FLCE_ERR_UNSUPPORTED;
    if ((ld * (i == 3 ? dw_esz : esz)) % 16 != 0) return FLCE_ERR_MISALIGNED;
  }
  // Tile ids are 32-bit: the largest grid (BT x V logits in 128 x 256 tiles,
  // up to 8 K splits) must stay below 2^31 work units.
  const int64_t bt_tiles = (p->BT + 127) / 128, v_tiles = (p->V + 255) / 256;
  if (bt_tiles > 0 && v_tiles > ((int64_t(1) << 28) - 1) / bt_tiles) return FLCE_ERR_UNSUPPORTED;
  // The fp32 CUDA-core kernels put 32-row blocks on gridDim.y (at most 65535).
  if (p->dtype == FLCE_FP32 && (p->BT + 31) / 32 > 65535) return FLCE_ERR_UNSUPPORTED;
  return FLCE_OK;
}

// Tensor-core GEMMs run on CTA pairs (256 x 256 tiles, tcgen05 cta_group::2)
// unless FLCE_CTA_PAIR=0 selects single-CTA 128 x 256 tiles.
bool use_pair() {
  static const bool v = [] {
    const char* e = std::getenv("FLCE_CTA_PAIR");
    return !(e && e[0] == '0');
  }();
  return v;
}

// Short-K CTA-pair GEMMs (H <= 1024: at most eight 128-deep stages per tile)
// run their exponential epilogues on eight warps, two per TMEM lane quarter,
// each of which keeps one (max, sum) partial per 128 columns; otherwise one
// partial per 256-column tile.  Returns log2 of the columns per partial.
int partial_shift(int64_t H) { return (use_pair() && H <= 1024) ? 7 : 8; }

#ifndef FLCE_PAIR_KSLICES
#define FLCE_PAIR_KSLICES 2
#endif
constexpr int kSlicesPair = FLCE_PAIR_KSLICES;
// CTA pairs the planner assumes (a B200 has 148 SMs); the split choice only
// affects speed, never results.
constexpr int kPlanPairs = 74;

// K splits for a GEMM of `tiles` pair tiles and `k_stages` pipeline stages:
// the split count whose work units fill the waves of `pairs` best, charging
// each extra split 1 % (its slab traffic and shorter pipelines); every split
// keeps at least 16 stages.
int pick_k_splits(int64_t tiles, int pairs, int64_t k_stages) {
  int best = 1;
  double best_t = double(cdiv(tiles, pairs));
  for (int sp = 2; sp <= 8; ++sp) {
    if (k_stages < 16 * sp) break;
    const double t = double(cdiv(tiles * sp, pairs)) / sp * (1.0 + 0.01 * (sp - 1));
    if (t < best_t) {
      best = sp;
      best_t = t;
    }
  }
  return best;
}

// Whether flce_fused runs the fused-in-forward schedule: bf16 only; chosen
// automatically once BT is large enough for two row chunks of >= 256 rows.
bool use_fused_forward(const flce_problem_t* p) {
  if (p->dtype != FLCE_BF16 || p->BT <= 0) return false;
  const int32_t s = g_schedule.load();
  if (s == 1) return false;
  if (s == 2) return true;
  return p->BT >= 512;
}

void make_plan_fused_forward(const flce_problem_t* p, Plan* pl) {
  const int64_t BT = p->BT, V = p->V, H = p->H;
  pl->BT = BT;
  pl->H = H;
  pl->V = V;
  pl->tc = true;
  pl->fused_fwd = true;
  pl->bn = 256;
  pl->part_shift = partial_shift(H);
  pl->part_tiles = cdiv(V, int64_t(1) << pl->part_shift);
  pl->ldp = round_up(V, 256);
  // At least two chunks once BT > 128, so the chunk buffer never holds the
  // whole BT x V; at most 1 GiB of q per chunk, or 2 GiB when the fp32 V x H
  // dW sum is itself above 1 GiB (then every extra chunk costs a multi-GB
  // read-modify-write pass over it).
  const bool big_dw = int64_t(V) * H * 4 > (int64_t(1) << 30);
  int64_t cmax = (int64_t(1) << (big_dw ? 31 : 30)) / (2 * pl->ldp) / 128 * 128;
  if (cmax < 128) cmax = 128;
  int64_t n = cdiv(BT, cmax);
  if (BT > 128 && n < 2) n = 2;
  // ... and chunks whose X rows (the forward GEMM's reused operand) stay
  // within 46 MiB, so they stay in L2 beside the streaming W and q: on the
  // Llama-3 shape a 67 MB chunk made the forward GEMM 7 % slower, and on
  // ragged BT from 12k to 34k rows chunks of 4224-5632 rows (this cap) beat
  // the memory cap's 6300-6900 by 1-3 %.
  const int64_t x_rows = (int64_t(46) << 20) / (2 * H) / 128 * 128;
  if (x_rows >= 128 && cdiv(BT, x_rows) > n) n = cdiv(BT, x_rows);
  pl->Cb = round_up(cdiv(BT, n), 128);
  pl->n_row_chunks = cdiv(BT, pl->Cb);
  size_t off = kHeaderBytes;
  const size_t rows = size_t(BT);
  pl->off_lse = off;
  off = align256(off + rows * 4);
  pl->off_target = off;
  off = align256(off + rows * 4);
  pl->off_rowloss = off;
  off = align256(off + rows * 4);
  pl->off_partial = off;
  off = align256(off + size_t(pl->part_tiles) * rows * 8);
  pl->off_p = off;
  off = align256(off + size_t(pl->Cb) * size_t(pl->ldp) * 2);
  // The fp32 running sum of dW over row chunks, unless dW itself is fp32.
  if (pl->n_row_chunks > 1 && !p->dw_fp32) {
    pl->off_dwacc = off;
    off = align256(off + size_t(V) * size_t(H) * 4);
  }
  pl->dx_splits = use_pair() ? pick_k_splits(cdiv(pl->Cb, 256) * cdiv(H, 256), kPlanPairs,
                                             cdiv(cdiv(V, 64), kSlicesPair))
                             : 1;
  if (pl->dx_splits > 1) {
    pl->off_dxslab = off;
    off = align256(off + size_t(pl->dx_splits) * size_t(pl->Cb) * size_t(H) * 4);
  }
  const size_t cb = size_t(pl->Cb);
  pl->off_xs = off;
  off = align256(off + cb * size_t(H) * 2);
  pl->off_ref = off;
  off = align256(off + cb * 4);
  pl->off_rowscale = off;
  off = align256(off + cb * 4);
  pl->off_flags = off;
  off = align256(off + size_t(cdiv(pl->Cb, kLseQRows)) * 4);
  pl->total = off;
}

void make_plan_base(const flce_problem_t* p, int op, Plan* pl, int64_t vc_max);
constexpr int kOpBackwardDxF32 = 32;

int64_t eff_ld(int64_t ld, int64_t H) { return ld == 0 ? H : ld; }

// Every schedule's plan, plus room for the shifted labels when the op
// shifts token ids itself.  Under the automatic schedule with a workspace
// cap, flce_fused takes the fused-in-forward plan only if it fits, else the
// recompute plan with the widest vocabulary chunk that fits.
void make_plan(const flce_problem_t* p, int op, Plan* pl) {
  const size_t extra = p->shift_seq_len > 0 ? align256(size_t(p->BT) * 8) : 0;
  const unsigned long long limit = g_schedule.load() == 0 ? g_ws_limit.load() : 0ull;
  make_plan_base(p, op, pl, 32768);
  if (limit && op == FLCE_OP_FUSED && p->dtype == FLCE_BF16 && pl->total + extra > limit) {
    for (int64_t vc = 32768; vc >= 256; vc /= 2) {
      *pl = Plan{};
      make_plan_base(p, FLCE_OP_FUSED + 16, pl, vc);  // the fused op, recompute schedule
      if (pl->total + extra <= limit) break;
    }
  }
  pl->dw_f32 = p->dw_fp32 && p->dtype == FLCE_BF16;
  pl->ldx = eff_ld(p->ldx, p->H);
  pl->ldw = eff_ld(p->ldw, p->H);
  pl->lddx = eff_ld(p->lddx, p->H);
  pl->lddw = eff_ld(p->lddw, p->H);
  if (p->shift_seq_len > 0) {
    pl->off_shift = pl->total;
    pl->total = align256(pl->total + size_t(p->BT) * 8);
  }
}

// op FLCE_OP_FUSED + 16 (internal): the fused op on the recompute schedule;
// kOpBackwardDxF32: the backward writing an fp32 dX that is its own running
// sum (no workspace for it).
void make_plan_base(const flce_problem_t* p, int op, Plan* pl, int64_t vc_max) {
  if (op == FLCE_OP_FUSED && use_fused_forward(p)) {
    make_plan_fused_forward(p, pl);
    return;
  }
  if (op == FLCE_OP_FUSED + 16) op = FLCE_OP_FUSED;
  const int op_in = op;
  if (op == kOpBackwardDxF32) op = FLCE_OP_BACKWARD;
  pl->BT = p->BT;
  pl->H = p->H;
  pl->V = p->V;
  pl->tc = p->dtype == FLCE_BF16;
  const int64_t BT = p->BT, V = p->V, H = p->H;
  const bool fwd = op == FLCE_OP_FORWARD || op == FLCE_OP_FUSED;
  const bool bwd = op == FLCE_OP_BACKWARD || op == FLCE_OP_FUSED;
  if (pl->tc) {
    pl->bn = 256;
    pl->part_shift = partial_shift(H);
    pl->part_tiles = cdiv(V, int64_t(1) << pl->part_shift);
    // Chunk width: G_c (BT x Vc bf16) kept at <= 512 MiB, Vc in [1024, 32768]
    // (narrower only under a workspace cap).
    int64_t vc = (int64_t(1) << 29) / (2 * (BT > 0 ? BT : 1));
    vc = vc / 256 * 256;
    if (vc < 1024) vc = 1024;
    if (vc > 32768) vc = 32768;
    if (vc > vc_max) vc = vc_max;
    pl->Vc = vc < round_up(V, 256) ? vc : round_up(V, 256);
    pl->g_elem = 2;
  } else {
    pl->bn = 32;
    pl->part_tiles = cdiv(V, 32);
    int64_t vc = (int64_t(1) << 28) / (4 * (BT > 0 ? BT : 1));
    vc = vc / 32 * 32;
    if (vc < 256) vc = 256;
    if (vc > 16384) vc = 16384;
    pl->Vc = vc < round_up(V, 32) ? vc : round_up(V, 32);
    pl->g_elem = 4;
  }
  pl->ldg = pl->Vc;
  pl->n_chunks = cdiv(V, pl->Vc);
  size_t off = kHeaderBytes;
  const size_t rows = size_t(BT > 0 ? BT : 1);
  if (op == FLCE_OP_FUSED) {
    pl->off_lse = off;
    off = align256(off + rows * 4);
  }
  if (fwd) {
    pl->off_target = off;
    off = align256(off + rows * 4);
    pl->off_rowloss = off;
    off = align256(off + rows * 4);
    pl->off_partial = off;
    off = align256(off + size_t(pl->part_tiles) * rows * 8);
  }
  if (bwd) {
    pl->off_g = off;
    off = align256(off + rows * size_t(pl->ldg) * pl->g_elem);
    if (pl->n_chunks > 1 && op_in != kOpBackwardDxF32) {
      pl->off_dxacc = off;
      off = align256(off + rows * size_t(H) * 4);
    }
  }
  pl->total = off;
}

// ----------------------------- tensor maps ---------------------------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// 2-D bf16 tensor [outer][inner] with row pitch row_bytes; box_inner x box_outer
// elements, 128-byte swizzle, zero fill outside the tensor.
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
              uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
              CUtensorMapDataType type = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, type, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// ------------------------------- launches ----------------------------------

TcShape make_shape(int64_t M, int64_t N, int64_t K, int bn, bool m_fast, int bm = kBM) {
  TcShape s{};
  s.M = int(M);
  s.N = int(N);
  s.K = int(K);
  s.m_tiles = int(cdiv(M, bm));
  s.n_tiles = int(cdiv(N, bn));
  s.k_blocks = int(cdiv(K, kBK));
  s.num_tiles = s.m_tiles * s.n_tiles;
  s.m_fast = m_fast ? 1 : 0;
  s.k_splits = 1;
  return s;
}

template <int BN, bool A_MN, bool B_MN, int MODE>
cudaError_t launch_tc(const CUtensorMap& a, const CUtensorMap& b, const TcShape& sh,
                      const TcEpi& ep, int num_sms, cudaStream_t st, int32_t kind_override = -1) {
  constexpr int32_t kind_default =
      (MODE == EPI_LSE || MODE == EPI_LSE_CAP) ? K_LSE_GEMM
      : (MODE == EPI_GRAD || MODE == EPI_GRAD_CAP) ? K_GRAD_GEMM
      : MODE == EPI_DX ? K_DX_GEMM : MODE == EPI_DW ? K_DW_GEMM : K_LSEQ_GEMM;
  const int32_t kind = kind_override >= 0 ? kind_override : kind_default;
  constexpr int STAGES = kStagesBN256;
  auto kern = tc_gemm_kernel<BN, A_MN, B_MN, MODE, STAGES>;
  constexpr uint32_t smem = TcSmem<BN, STAGES>::kTotal;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  if (sh.num_tiles <= 0) return cudaSuccess;
  const int grid = sh.num_tiles < num_sms ? sh.num_tiles : num_sms;
  prof_before(st);
  kern<<<grid, kTcThreads, smem, st>>>(a, b, sh, ep);
  prof_after(st, kind);
  return cudaGetLastError();
}

// Rows of B's K-major TMA box: each CTA of a pair loads 128 of the 256.
uint32_t b_box_rows() { return use_pair() ? 128u : 256u; }

#ifndef FLCE_PAIR_STAGES
#define FLCE_PAIR_STAGES 3
#endif
constexpr int kStagesPair = FLCE_PAIR_STAGES;

template <bool A_MN, bool B_MN, int MODE, int EW>
cudaError_t launch_tc2(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& c,
                       const TcShape& sh, const TcEpi& ep, int num_sms, cudaStream_t st,
                       int32_t kind) {
  auto kern = tc2_gemm_kernel<A_MN, B_MN, MODE, kStagesPair, kSlicesPair, EW>;
  constexpr uint32_t smem = Tc2Smem<kStagesPair, kSlicesPair>::kTotal;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  if (sh.num_tiles <= 0) return cudaSuccess;
  // Persistent grid: as many pairs as can be resident at once (tiles are
  // assigned statically, so a pair that had to wait would serialise its share).
  static int max_pairs = -1;
  if (max_pairs < 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(num_sms & ~1), 1, 1);
    cfg.blockDim = dim3(tc2_threads(EW), 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 2;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    max_pairs = (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) == cudaSuccess && n > 0)
                    ? n : num_sms / 2;
  }
  int pairs = num_sms / 2 < max_pairs ? num_sms / 2 : max_pairs;
  if (sh.num_tiles * sh.k_splits < pairs) pairs = sh.num_tiles * sh.k_splits;
  prof_before(st);
  kern<<<2 * pairs, tc2_threads(EW), smem, st>>>(a, b, c, sh, ep);
  prof_after(st, kind);
  return cudaGetLastError();
}

struct GemmArgs {
  int64_t M, N, K;
  bool m_fast;
  int a_mn_off = 0, a_k_off = 0, b_mn_off = 0, b_k_off = 0;
  int k_splits = 1;  // CTA-pair kernels only (EPI_DX slabs)
  bool wide_epi = false;  // CTA pairs: eight epilogue warps for the exponential epilogues
};

// `c` is the TMA map of the bf16 output the CTA-pair epilogue stores (q, G,
// dW, or dX in a single pass); boxes of 64 columns x 32 rows.  Modes without
// such an output pass any valid map.
template <bool A_MN, bool B_MN, int MODE>
cudaError_t launch_gemm(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& c,
                        const GemmArgs& g, const TcEpi& ep, int num_sms, cudaStream_t st,
                        int32_t kind = -1) {
  constexpr int32_t kind_default =
      (MODE == EPI_LSE || MODE == EPI_LSE_CAP) ? K_LSE_GEMM
      : (MODE == EPI_GRAD || MODE == EPI_GRAD_CAP) ? K_GRAD_GEMM
      : MODE == EPI_DX ? K_DX_GEMM : MODE == EPI_DW ? K_DW_GEMM : K_LSEQ_GEMM;
  if (kind < 0) kind = kind_default;
  const bool pair = use_pair();
  TcShape sh = make_shape(g.M, g.N, g.K, 256, g.m_fast, pair ? kPairBM : kBM);
  sh.a_mn_off = g.a_mn_off;
  sh.a_k_off = g.a_k_off;
  sh.b_mn_off = g.b_mn_off;
  sh.b_k_off = g.b_k_off;
  sh.k_splits = pair ? g.k_splits : 1;
  if (pair) {
    // Eight epilogue warps for the split-K dX slabs, and for the exponential
    // epilogues when the caller asks (short K: the epilogue, not the MMA,
    // paces the tile); four for the fp32 running sums, single-pass dX and dW,
    // and the exponential epilogues of long-K GEMMs, which measured faster so.
    if constexpr (MODE == EPI_DW) {
      return launch_tc2<A_MN, B_MN, MODE, 4>(a, b, c, sh, ep, num_sms, st, kind);
    } else if constexpr (MODE == EPI_DX) {
      if (sh.k_splits == 1)
        return launch_tc2<A_MN, B_MN, MODE, 4>(a, b, c, sh, ep, num_sms, st, kind);
      return launch_tc2<A_MN, B_MN, MODE, 8>(a, b, c, sh, ep, num_sms, st, kind);
    } else {
      if (g.wide_epi) return launch_tc2<A_MN, B_MN, MODE, 8>(a, b, c, sh, ep, num_sms, st, kind);
      return launch_tc2<A_MN, B_MN, MODE, 4>(a, b, c, sh, ep, num_sms, st, kind);
    }
  }
  return launch_tc<256, A_MN, B_MN, MODE>(a, b, sh, ep, num_sms, st, kind);
}

struct Ptrs {
  const void* X;
  const void* W;
  const int64_t* labels;
  float* loss;
  float* lse;          // forward output / backward input
  const float* dloss_dev;
  float dloss_host;
  void* dX;
  void* dW;
  uint8_t* ws;
  const int64_t* n_valid_global = nullptr;  // device count over all ranks, or null
  // dW handed over in vocabulary slices: event s recorded once rows
  // [s * slice_rows, (s + 1) * slice_rows) of dW are final (none: 0 / null)
  int32_t n_slices = 0;
  cudaEvent_t* slice_done = nullptr;
};

// Rows of dW per slice when dW is handed over in n vocabulary slices: the
// slices are [s * r, min(V, (s + 1) * r)) with r a multiple of 256 (whole
// GEMM tiles), so some trailing slices may be empty.
int64_t dw_slice_rows(int64_t V, int32_t n) { return round_up(cdiv(V, int64_t(n)), 256); }

// Record every slice's event at once (paths whose dW is final only at the end).
flce_status_t record_all_slices(const Ptrs& q, cudaStream_t st) {
  for (int32_t s = 0; s < q.n_slices; ++s)
    if (cudaEventRecord(q.slice_done[s], st) != cudaSuccess) return FLCE_ERR_CUDA;
  return FLCE_OK;
}

TcEpi base_epi(const flce_problem_t* p, const Plan& pl, const Ptrs& q) {
  TcEpi e{};
  e.status = reinterpret_cast<int*>(q.ws);
  e.wait_limit_ns = g_wait_limit_ns.load();
  e.labels = q.labels;
  e.ignore_index = p->ignore_index;
  e.BT = pl.BT;
  e.V = pl.V;
  e.H = pl.H;
  e.softcap = softcap_on(p->softcap) ? p->softcap : 0.f;
  e.ld_dx = pl.lddx;
  e.ld_dw = pl.lddw;
  e.ld_acc = pl.H;
  e.label_off = pl.label_off;
  return e;
}

SimtEpi base_simt(const flce_problem_t* p, const Plan& pl, const Ptrs& q) {
  SimtEpi e{};
  e.hdr = reinterpret_cast<const WsHeader*>(q.ws);
  e.labels = q.labels;
  e.ignore_index = p->ignore_index;
  e.BT = pl.BT;
  e.H = pl.H;
  e.V = pl.V;
  e.softcap = softcap_on(p->softcap) ? p->softcap : 0.f;
  e.ldx = pl.ldx;
  e.ldw = pl.ldw;
  e.lddx = pl.lddx;
  e.lddw = pl.lddw;
  e.label_off = pl.label_off;
  return e;
}

int device_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

flce_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? FLCE_OK : FLCE_ERR_CUDA; }

#define FLCE_TRY(expr)                                  \
  do {                                                  \
    cudaError_t e_ = (expr);                            \
    if (e_ != cudaSuccess) return FLCE_ERR_CUDA;        \
  } while (0)

// With shift_seq_len > 0, q.labels (token ids) is replaced by the op's own
// shifted copy in the workspace before anything reads it.
flce_status_t enqueue_shift(const flce_problem_t* p, const Plan& pl, Ptrs* q, cudaStream_t st) {
  if (p->shift_seq_len <= 0) return FLCE_OK;
  int64_t* out = reinterpret_cast<int64_t*>(q->ws + pl.off_shift);
  if (p->BT > 0) {
    int blocks = int(cdiv(p->BT, 256));
    if (blocks > 1024) blocks = 1024;
    prof_before(st);
    shift_labels_kernel<<<blocks, 256, 0, st>>>(q->labels, p->BT, p->shift_seq_len,
                                                p->ignore_index, out);
    prof_after(st, K_SHIFT_LABELS);
    FLCE_TRY(cudaGetLastError());
  }
  q->labels = out;
  return FLCE_OK;
}

flce_status_t enqueue_labels(const flce_problem_t* p, const Ptrs& q, cudaStream_t st) {
  prof_before(st);
  labels_kernel<<<1, 1024, 0, st>>>(q.labels, p->BT, p->V, p->ignore_index,
                                    reinterpret_cast<WsHeader*>(q.ws));
  prof_after(st, K_LABELS);
  FLCE_TRY(cudaGetLastError());
  if (q.n_valid_global) {
    prof_before(st);
    set_n_valid_kernel<<<1, 1, 0, st>>>(reinterpret_cast<WsHeader*>(q.ws), q.n_valid_global);
    prof_after(st, K_SET_NVALID);
    FLCE_TRY(cudaGetLastError());
  }
  return FLCE_OK;
}

flce_status_t enqueue_forward(const flce_problem_t* p, const Plan& pl, const Ptrs& q,
                              cudaStream_t st) {
  const int64_t BT = pl.BT, V = pl.V, H = pl.H;
  WsHeader* hdr = reinterpret_cast<WsHeader*>(q.ws);
  float2* partial = reinterpret_cast<float2*>(q.ws + pl.off_partial);
  float* target = reinterpret_cast<float*>(q.ws + pl.off_target);
  float* rowloss = reinterpret_cast<float*>(q.ws + pl.off_rowloss);
  if (BT > 0) {
    if (pl.tc) {
      CUtensorMap ma, mb;
      if (!make_map(&ma, q.X, H, BT, pl.ldx * 2, 64, kBM)) return FLCE_ERR_CUDA;
      if (!make_map(&mb, q.W, H, V, pl.ldw * 2, 64, b_box_rows())) return FLCE_ERR_CUDA;
      TcEpi ep = base_epi(p, pl, q);
      ep.partial = partial;
      ep.target = target;
      GemmArgs g{BT, V, H, true};
      g.wide_epi = pl.part_shift == 7;
      if (ep.softcap > 0.f)
        FLCE_TRY((launch_gemm<false, false, EPI_LSE_CAP>(ma, mb, ma, g, ep, device_sms(), st)));
      else
        FLCE_TRY((launch_gemm<false, false, EPI_LSE>(ma, mb, ma, g, ep, device_sms(), st)));
    } else {
      SimtEpi ep = base_simt(p, pl, q);
      ep.partial = partial;
      ep.target = target;
      dim3 grid(unsigned(cdiv(V, 32)), unsigned(cdiv(BT, 32)));
      prof_before(st);
      simt_logits_kernel<float, 0><<<grid, dim3(32, 8), 0, st>>>(
          static_cast<const float*>(q.X), static_cast<const float*>(q.W), ep);
      prof_after(st, K_SIMT_LOGITS);
      FLCE_TRY(cudaGetLastError());
    }
    prof_before(st);
    combine_kernel<<<unsigned(cdiv(BT, 256)), 256, 0, st>>>(
        partial, int(pl.part_tiles), BT, target, q.labels, p->ignore_index, q.lse, rowloss, hdr);
    prof_after(st, K_COMBINE);
    FLCE_TRY(cudaGetLastError());
  }
  prof_before(st);
  finalize_kernel<<<1, 1024, 0, st>>>(rowloss, BT, hdr, q.loss);
  prof_after(st, K_FINALIZE);
  return cuda_status(cudaGetLastError());
}

flce_status_t enqueue_backward(const flce_problem_t* p, const Plan& pl, const Ptrs& q,
                               cudaStream_t st) {
  const int64_t BT = pl.BT, V = pl.V, H = pl.H;
  const size_t esz = (pl.tc && !pl.dw_f32) ? 2 : 4;  // dW's element size
  if (BT == 0) {
    prof_before(st);
    FLCE_TRY(cudaMemset2DAsync(q.dW, size_t(pl.lddw) * esz, 0, size_t(H) * esz, size_t(V), st));
    prof_after(st, K_MEMSET);
    return FLCE_OK;
  }
  const long long* n_valid =
      reinterpret_cast<const long long*>(q.ws + offsetof(WsHeader, n_valid));
  if (pl.tc) {
    __nv_bfloat16* G = reinterpret_cast<__nv_bfloat16*>(q.ws + pl.off_g);
    CUtensorMap mx_k, mw_k, mg_k, mw_mn, mg_mn, mx_mn, mg_out, mdx_out;
    bool ok = make_map(&mg_out, G, pl.ldg, BT, pl.ldg * 2, 64, 32) &&
              (pl.dx_f32 ? make_map(&mdx_out, q.dX, H, BT, pl.lddx * 4, 32, 32,
                                    CU_TENSOR_MAP_DATA_TYPE_FLOAT32)
                         : make_map(&mdx_out, q.dX, H, BT, pl.lddx * 2, 64, 32)) &&
              make_map(&mx_k, q.X, H, BT, pl.ldx * 2, 64, kBM) &&
              make_map(&mw_k, q.W, H, V, pl.ldw * 2, 64, b_box_rows()) &&
              make_map(&mg_k, G, pl.ldg, BT, pl.ldg * 2, 64, kBM) &&
              make_map(&mw_mn, q.W, H, V, pl.ldw * 2, 64, 64) &&
              make_map(&mg_mn, G, pl.ldg, BT, pl.ldg * 2, 64, 64) &&
              make_map(&mx_mn, q.X, H, BT, pl.ldx * 2, 64, 64);
    if (!ok) return FLCE_ERR_CUDA;
    const int sms = device_sms();
    for (int64_t c = 0; c < pl.n_chunks; ++c) {
      const int64_t v0 = c * pl.Vc;
      const int64_t width = (V - v0) < pl.Vc ? (V - v0) : pl.Vc;
      TcEpi ep = base_epi(p, pl, q);
      ep.lse = q.lse;
      ep.dloss_dev = q.dloss_dev;
      ep.dloss_host = q.dloss_host;
      ep.n_valid = n_valid;
      ep.G = G;
      ep.ldg = pl.ldg;
      ep.v0 = v0;
      // the fp32 running sum of dX over vocabulary chunks: the workspace, or
      // the fp32 dX itself
      ep.dx_acc = pl.dx_f32 ? static_cast<float*>(q.dX)
                            : reinterpret_cast<float*>(q.ws + pl.off_dxacc);
      ep.ld_acc = pl.dx_f32 ? pl.lddx : H;
      ep.dx = static_cast<__nv_bfloat16*>(q.dX);
      ep.dx_first = c == 0;
      ep.dx_last = c == pl.n_chunks - 1;
      ep.dw = static_cast<__nv_bfloat16*>(q.dW);
      // G_c = softmax-grad of the recomputed logits X W_c^T
      GemmArgs gg{BT, round_up(width, 256), H, true};
      gg.wide_epi = pl.part_shift == 7;
      gg.b_mn_off = int(v0);
      TcEpi eg = ep;
      eg.out_cols = int(pl.ldg);
      if (eg.softcap > 0.f)
        FLCE_TRY((launch_gemm<false, false, EPI_GRAD_CAP>(mx_k, mw_k, mg_out, gg, eg, sms, st)));
      else
        FLCE_TRY((launch_gemm<false, false, EPI_GRAD>(mx_k, mw_k, mg_out, gg, eg, sms, st)));
      // dX (+)= G_c W_c    (K = chunk columns)
      GemmArgs gx{BT, H, round_up(width, 64), false};
      gx.b_k_off = int(v0);
      TcEpi ex = ep;
      ex.out_cols = int(H);
      ex.out_f32 = pl.dx_f32 ? 1 : 0;
      FLCE_TRY((launch_gemm<false, true, EPI_DX>(mg_k, mw_mn, mdx_out, gx, ex, sms, st)));
      // dW_c = G_c^T X     (K = BT); the output map ends at the chunk's last row
      CUtensorMap mdw_out;
      const bool ok_dw =
          pl.dw_f32 ? make_map(&mdw_out, q.dW, H, v0 + width, pl.lddw * 4, 32, 32,
                               CU_TENSOR_MAP_DATA_TYPE_FLOAT32)
                    : make_map(&mdw_out, q.dW, H, v0 + width, pl.lddw * 2, 64, 32);
      if (!ok_dw) return FLCE_ERR_CUDA;
      TcEpi ewo = ep;
      ewo.out_row_off = int(v0);
      ewo.out_cols = int(H);
      ewo.out_f32 = pl.dw_f32 ? 1 : 0;
      ewo.dw32 = static_cast<float*>(q.dW);
      GemmArgs gw{width, H, BT, false};
      FLCE_TRY((launch_gemm<true, true, EPI_DW>(mg_mn, mx_mn, mdw_out, gw, ewo, sms, st)));
    }
  } else {
    float* G = reinterpret_cast<float*>(q.ws + pl.off_g);
    for (int64_t c = 0; c < pl.n_chunks; ++c) {
      const int64_t v0 = c * pl.Vc;
      const int64_t width = (V - v0) < pl.Vc ? (V - v0) : pl.Vc;
      SimtEpi ep = base_simt(p, pl, q);
      ep.lse = q.lse;
      ep.dloss_dev = q.dloss_dev;
      ep.dloss_host = q.dloss_host;
      ep.G = G;
      ep.ldg = pl.ldg;
      ep.v0 = v0;
      ep.chunk = width;
      ep.dx_acc = reinterpret_cast<float*>(q.ws + pl.off_dxacc);
      ep.dx = q.dX;
      ep.dx_first = c == 0;
      ep.dx_last = c == pl.n_chunks - 1;
      ep.dw = q.dW;
      const float* X = static_cast<const float*>(q.X);
      const float* W = static_cast<const float*>(q.W);
      prof_before(st);
      simt_logits_kernel<float, 1><<<dim3(unsigned(cdiv(width, 32)), unsigned(cdiv(BT, 32))),
                                     dim3(32, 8), 0, st>>>(X, W, ep);
      prof_after(st, K_SIMT_GRAD);
      prof_before(st);
      simt_gemm_kernel<float, 2><<<dim3(unsigned(cdiv(H, 32)), unsigned(cdiv(BT, 32))),
                                   dim3(32, 8), 0, st>>>(W, ep);
      prof_after(st, K_SIMT_DX);
      prof_before(st);
      simt_gemm_kernel<float, 3><<<dim3(unsigned(cdiv(H, 32)), unsigned(cdiv(width, 32))),
                                   dim3(32, 8), 0, st>>>(X, ep);
      prof_after(st, K_SIMT_DW);
      FLCE_TRY(cudaGetLastError());
    }
  }
  return FLCE_OK;
}

// flce_fused, fused-in-forward schedule (6*BT*H*V FLOP: no logit recompute).
// For each chunk of Cb rows:
//   lse_q GEMM   X_b W^T; epilogue stores q = exp(y - R) dy/dz (bf16) into P
//                with one reference R per row (0), the (max, sum) partials
//                and the target logit
//   lse_q pass 1 lse, NLL, f = 1 / sum and the dX factor per row; the label
//                column of P patched so that G = (dloss / N) diag(f) P;
//                Xs = bf16(f X_b).  Rows whose logits leave the range R = 0
//                serves are flagged instead
//   repair GEMM  the forward GEMM again, only for the flagged 32-row groups,
//                against each row's exact maximum (returns at once when
//                nothing is flagged)
//   lse_q pass 2 the flagged rows as in pass 1
//   dX GEMM      dX_b = f (dloss / N) (P W)   (K = all of V; bf16 out)
//   dW GEMM      dW  (+)= (dloss / N) P^T Xs  (fp32 running sum over chunks,
//                bf16 -- or the fp32 sum -- on the last chunk)
// then the loss over all rows.  P is never rewritten in full: the only pass
// over it besides the two GEMMs that read it is one bf16 store per row.
// Labels were checked by the caller.
flce_status_t enqueue_fused_forward(const flce_problem_t* p, const Plan& pl, const Ptrs& q,
                                    cudaStream_t st) {
  const int64_t BT = pl.BT, V = pl.V, H = pl.H;
  WsHeader* hdr = reinterpret_cast<WsHeader*>(q.ws);
  float2* partial = reinterpret_cast<float2*>(q.ws + pl.off_partial);
  float* target = reinterpret_cast<float*>(q.ws + pl.off_target);
  float* rowloss = reinterpret_cast<float*>(q.ws + pl.off_rowloss);
  float* lse = reinterpret_cast<float*>(q.ws + pl.off_lse);
  __nv_bfloat16* P = reinterpret_cast<__nv_bfloat16*>(q.ws + pl.off_p);
  __nv_bfloat16* Xs = reinterpret_cast<__nv_bfloat16*>(q.ws + pl.off_xs);
  float* ref = reinterpret_cast<float*>(q.ws + pl.off_ref);
  float* row_scale = reinterpret_cast<float*>(q.ws + pl.off_rowscale);
  int* flags = reinterpret_cast<int*>(q.ws + pl.off_flags);
  CUtensorMap mx_k, mw_k, mw_mn, mdw_out;
  // dW's map: bf16 pieces of 64 columns, or fp32 pieces of 32 when dW is fp32
  const bool ok_dw = pl.dw_f32 ? make_map(&mdw_out, q.dW, H, V, pl.lddw * 4, 32, 32,
                                          CU_TENSOR_MAP_DATA_TYPE_FLOAT32)
                               : make_map(&mdw_out, q.dW, H, V, pl.lddw * 2, 64, 32);
  if (!(ok_dw &&
        make_map(&mx_k, q.X, H, BT, pl.ldx * 2, 64, kBM) &&
        make_map(&mw_k, q.W, H, V, pl.ldw * 2, 64, b_box_rows()) &&
        make_map(&mw_mn, q.W, H, V, pl.ldw * 2, 64, 64)))
    return FLCE_ERR_CUDA;
  const int sms = device_sms();
  const float cap = softcap_on(p->softcap) ? p->softcap : 0.f;
  for (int64_t b = 0; b < pl.n_row_chunks; ++b) {
    const int64_t row0 = b * pl.Cb;
    const int64_t rows = (BT - row0) < pl.Cb ? (BT - row0) : pl.Cb;
    CUtensorMap mp_k, mp_mn, mp_out, mdx_out, mxs_mn;
    if (!(make_map(&mp_k, P, pl.ldp, rows, pl.ldp * 2, 64, kBM) &&
          make_map(&mp_mn, P, pl.ldp, rows, pl.ldp * 2, 64, 64) &&
          make_map(&mp_out, P, pl.ldp, rows, pl.ldp * 2, 64, 32) &&
          make_map(&mxs_mn, Xs, H, rows, H * 2, 64, 64) &&
          make_map(&mdx_out, static_cast<__nv_bfloat16*>(q.dX) + row0 * pl.lddx, H, rows,
                   pl.lddx * 2, 64, 32)))
      return FLCE_ERR_CUDA;
    TcEpi ep = base_epi(p, pl, q);
    ep.partial = partial;
    ep.target = target;
    ep.row0 = row0;
    ep.P = P;
    ep.ldp = pl.ldp;
    ep.out_cols = int(pl.ldp);
    GemmArgs gf{rows, V, H, true};
    gf.wide_epi = pl.part_shift == 7;
    gf.a_mn_off = int(row0);
    const unsigned groups = unsigned(cdiv(rows, kLseQRows));
    for (int pass = 1; pass <= 2; ++pass) {
      TcEpi ef = ep;
      if (pass == 2) {  // recompute only the flagged row groups
        ef.ref = ref;
        ef.row_group_flags = flags;
        ef.n_groups = int(groups);
      }
      const int32_t kind = pass == 1 ? K_LSEQ_GEMM : K_LSEQ_REPAIR;
      if (ef.softcap > 0.f)
        FLCE_TRY((launch_gemm<false, false, EPI_LSE_Q_CAP>(mx_k, mw_k, mp_out, gf, ef, sms, st,
                                                           kind)));
      else
        FLCE_TRY((launch_gemm<false, false, EPI_LSE_Q>(mx_k, mw_k, mp_out, gf, ef, sms, st,
                                                       kind)));
      prof_before(st);
      lse_q_kernel<<<groups, kLseQThreads, 0, st>>>(
          pass, partial, int(pl.part_tiles), BT, row0, rows, target, q.labels, p->ignore_index, P,
          pl.ldp, static_cast<const __nv_bfloat16*>(q.X), pl.ldx, H, Xs, ref, flags, lse,
          rowloss, row_scale, hdr, q.dloss_host, cap);
      prof_after(st, K_LSEQ);
      FLCE_TRY(cudaGetLastError());
    }
    // dX rows of this chunk: K runs over the whole vocabulary; each row
    // scaled by its f dloss / N
    TcEpi ex = ep;
    ex.dx = static_cast<__nv_bfloat16*>(q.dX) + row0 * pl.lddx;
    ex.dx_first = 1;
    ex.dx_last = 1;
    ex.dx_acc = reinterpret_cast<float*>(q.ws + pl.off_dxslab);
    ex.slab_stride = pl.Cb * H;
    ex.out_cols = int(H);
    ex.row_scale = row_scale;
    GemmArgs gx{rows, H, round_up(V, 64), false};
    gx.k_splits = pl.dx_splits;
    FLCE_TRY((launch_gemm<false, true, EPI_DX>(mp_k, mw_mn, mdx_out, gx, ex, sms, st)));
    if (pl.dx_splits > 1) {
      const int64_t n = rows * H;
      int blocks = int(cdiv(n, 8 * 256));
      if (blocks > 8 * sms) blocks = 8 * sms;
      prof_before(st);
      slab_reduce_kernel<<<blocks, 256, 0, st>>>(ex.dx_acc, pl.dx_splits, ex.slab_stride, n, H,
                                                 ex.dx, pl.lddx, row_scale, hdr);
      prof_after(st, K_DX_REDUCE);
      FLCE_TRY(cudaGetLastError());
    }
    // dW += (dloss / N) P^T Xs: an fp32 running sum over the row chunks, in
    // the workspace, or in dW itself when dW is fp32
    TcEpi ew = ep;
    ew.dx_acc = pl.dw_f32 ? static_cast<float*>(q.dW)
                          : reinterpret_cast<float*>(q.ws + pl.off_dwacc);
    ew.ld_acc = pl.dw_f32 ? pl.lddw : H;
    ew.out_f32 = pl.dw_f32 ? 1 : 0;
    ew.dx = static_cast<__nv_bfloat16*>(q.dW);
    ew.ld_dx = pl.lddw;
    ew.dx_first = b == 0;
    ew.dx_last = b == pl.n_row_chunks - 1;
    ew.out_cols = int(H);
    ew.scale_by_nvalid = 1;
    ew.n_valid = reinterpret_cast<const long long*>(q.ws + offsetof(WsHeader, n_valid));
    ew.dloss_host = q.dloss_host;
    // The sum goes out by TMA stores: fp32 rows of the running sum, then dW
    // on the last chunk (bf16, or the fp32 sum itself).
    ew.tma_rmw = 1;
    CUtensorMap macc;
    if (!ew.dx_last && !make_map(&macc, ew.dx_acc, H, V, size_t(ew.ld_acc) * 4, 32, 32,
                                 CU_TENSOR_MAP_DATA_TYPE_FLOAT32))
      return FLCE_ERR_CUDA;
    if (ew.dx_last && q.n_slices > 0) {
      // The last chunk's dW GEMM in vocabulary slices, each slice's rows of
      // dW final when its launch ends: the same GEMM with M = the slice's
      // rows, the A operand (P^T) offset to the slice's first column and the
      // outputs' base pointers to its first row.
      const int64_t vs = dw_slice_rows(V, q.n_slices);
      for (int32_t sl = 0; sl < q.n_slices; ++sl) {
        const int64_t v0 = int64_t(sl) * vs;
        if (v0 < V) {
          const int64_t vn = (V - v0) < vs ? (V - v0) : vs;
          TcEpi es = ew;
          es.dx_acc = ew.dx_acc + v0 * ew.ld_acc;
          if (!pl.dw_f32) es.dx = ew.dx + v0 * pl.lddw;
          CUtensorMap mo;
          const bool ok = pl.dw_f32
                              ? make_map(&mo, static_cast<float*>(q.dW) + v0 * pl.lddw, H, vn,
                                         pl.lddw * 4, 32, 32, CU_TENSOR_MAP_DATA_TYPE_FLOAT32)
                              : make_map(&mo, static_cast<__nv_bfloat16*>(q.dW) + v0 * pl.lddw,
                                         H, vn, pl.lddw * 2, 64, 32);
          if (!ok) return FLCE_ERR_CUDA;
          GemmArgs gs{vn, H, rows, false};
          gs.a_mn_off = int(v0);
          FLCE_TRY((launch_gemm<true, true, EPI_DX>(mp_mn, mxs_mn, mo, gs, es, sms, st,
                                                    K_DWACC_GEMM)));
        }
        if (cudaEventRecord(q.slice_done[sl], st) != cudaSuccess) return FLCE_ERR_CUDA;
      }
    } else {
      GemmArgs gw{V, H, rows, false};
      FLCE_TRY((launch_gemm<true, true, EPI_DX>(mp_mn, mxs_mn, ew.dx_last ? mdw_out : macc, gw,
                                                ew, sms, st, K_DWACC_GEMM)));
    }
  }
  prof_before(st);
  finalize_kernel<<<1, 1024, 0, st>>>(rowloss, BT, hdr, q.loss);
  prof_after(st, K_FINALIZE);
  return cuda_status(cudaGetLastError());
}

bool aligned(const void* ptr, size_t a) { return (reinterpret_cast<uintptr_t>(ptr) % a) == 0; }

// The epilogues' own approximations beside CUDA's functions, for a bound
// test: out[4i..4i+3] = tanh_fast(x), tanhf(x), ex2a(x), exp2f(x).
__global__ void approx_selftest_kernel(const float* __restrict__ x, int64_t n,
                                       float* __restrict__ out) {
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += int64_t(gridDim.x) * blockDim.x) {
    const float v = x[i];
    out[4 * i] = tanh_fast(v);
    out[4 * i + 1] = tanhf(v);
    out[4 * i + 2] = ex2a(v);
    out[4 * i + 3] = exp2f(v);
  }
}

flce_status_t check_common(const flce_problem_t* p, const void* X, const void* W,
                           const int64_t* labels, void* ws) {
  if (p->BT > 0 && (!X || !labels)) return FLCE_ERR_INVALID_ARG;
  if (!W || !ws) return FLCE_ERR_INVALID_ARG;
  if (!aligned(X, 16) || !aligned(W, 16) || !aligned(labels, 8) || !aligned(ws, 256))
    return FLCE_ERR_MISALIGNED;
  return FLCE_OK;
}

}  // namespace

// ------------------------- shared with flce_ce.cu ---------------------------

namespace flce_internal {

void prof_before(cudaStream_t st) { ::prof_before(st); }
void prof_after(cudaStream_t st, int32_t kind) { ::prof_after(st, kind); }
void reset_launch_count() { t_launches = 0; }
unsigned long long wait_limit_ns() { return g_wait_limit_ns.load(); }
int device_sm_count() { return device_sms(); }

cudaError_t launch_labels(const int64_t* labels, int64_t BT, int64_t V, int64_t ignore_index,
                          void* ws, cudaStream_t st) {
  ::prof_before(st);
  labels_kernel<<<1, 1024, 0, st>>>(labels, BT, V, ignore_index, static_cast<WsHeader*>(ws));
  ::prof_after(st, K_LABELS);
  return cudaGetLastError();
}

cudaError_t launch_shift(const int64_t* ids, int64_t BT, int64_t T, int64_t ignore_index,
                         int64_t* out, cudaStream_t st) {
  if (BT <= 0) return cudaSuccess;
  int blocks = int(cdiv(BT, 256));
  if (blocks > 1024) blocks = 1024;
  ::prof_before(st);
  shift_labels_kernel<<<blocks, 256, 0, st>>>(ids, BT, T, ignore_index, out);
  ::prof_after(st, K_SHIFT_LABELS);
  return cudaGetLastError();
}

cudaError_t launch_finalize(const float* row_loss, int64_t BT, const void* ws, float* loss,
                            cudaStream_t st) {
  ::prof_before(st);
  finalize_kernel<<<1, 1024, 0, st>>>(row_loss, BT, static_cast<const WsHeader*>(ws), loss);
  ::prof_after(st, K_FINALIZE);
  return cudaGetLastError();
}

}  // namespace flce_internal

// ------------------------------- C ABI -------------------------------------

extern "C" {

size_t flce_workspace_size(const flce_problem_t* p, int op) {
  if (check_problem(p) != FLCE_OK) return 0;
  if (op != FLCE_OP_FORWARD && op != FLCE_OP_BACKWARD && op != FLCE_OP_FUSED) return 0;
  Plan pl;
  make_plan(p, op, &pl);
  return pl.total;
}

flce_status_t flce_forward(const flce_problem_t* p, const void* X, const void* W,
                           const int64_t* labels, float* loss, float* lse, void* ws,
                           size_t ws_bytes, struct CUstream_st* stream) {
  t_launches = 0;
  flce_status_t s = check_problem(p);
  if (s != FLCE_OK) return s;
  if ((s = check_common(p, X, W, labels, ws)) != FLCE_OK) return s;
  if (!loss || (p->BT > 0 && !lse)) return FLCE_ERR_INVALID_ARG;
  if (!aligned(loss, 4) || !aligned(lse, 4)) return FLCE_ERR_MISALIGNED;
  Plan pl;
  make_plan(p, FLCE_OP_FORWARD, &pl);
  if (ws_bytes < pl.total) return FLCE_ERR_WORKSPACE_TOO_SMALL;
  Ptrs q{X, W, labels, loss, lse, nullptr, 1.f, nullptr, nullptr, static_cast<uint8_t*>(ws)};
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if ((s = enqueue_shift(p, pl, &q, st)) != FLCE_OK) return s;
  if ((s = enqueue_labels(p, q, st)) != FLCE_OK) return s;
  return enqueue_forward(p, pl, q, st);
}

flce_status_t flce_backward(const flce_problem_t* p, const void* X, const void* W,
                            const int64_t* labels, const float* lse, const float* dloss,
                            void* dX, void* dW, void* ws, size_t ws_bytes,
                            struct CUstream_st* stream) {
  t_launches = 0;
  flce_status_t s = check_problem(p);
  if (s != FLCE_OK) return s;
  if ((s = check_common(p, X, W, labels, ws)) != FLCE_OK) return s;
  if (!dloss || !dW || (p->BT > 0 && (!lse || !dX))) return FLCE_ERR_INVALID_ARG;
  if (!aligned(dX, 16) || !aligned(dW, 16) || !aligned(lse, 4) || !aligned(dloss, 4))
    return FLCE_ERR_MISALIGNED;
  Plan pl;
  make_plan(p, FLCE_OP_BACKWARD, &pl);
  if (ws_bytes < pl.total) return FLCE_ERR_WORKSPACE_TOO_SMALL;
  Ptrs q{X, W, labels, nullptr, const_cast<float*>(lse), dloss, 1.f, dX, dW,
         static_cast<uint8_t*>(ws)};
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if ((s = enqueue_shift(p, pl, &q, st)) != FLCE_OK) return s;
  if ((s = enqueue_labels(p, q, st)) != FLCE_OK) return s;
  return enqueue_backward(p, pl, q, st);
}

static flce_status_t fused_impl(const flce_problem_t* p, const void* X, const void* W,
                         const int64_t* labels, const int64_t* n_valid_global, float dloss,
                         float* loss, void* dX, void* dW, void* ws, size_t ws_bytes,
                         struct CUstream_st* stream, int32_t n_slices = 0,
                         struct CUevent_st* const* slice_done = nullptr) {
  t_launches = 0;
  flce_status_t s = check_problem(p);
  if (s != FLCE_OK) return s;
  if (n_slices < 0 || n_slices > kMaxDwSlices || (n_slices > 0 && !slice_done))
    return FLCE_ERR_INVALID_ARG;
  for (int32_t i = 0; i < n_slices; ++i)
    if (!slice_done[i]) return FLCE_ERR_INVALID_ARG;
  if ((s = check_common(p, X, W, labels, ws)) != FLCE_OK) return s;
  if (!loss || !dW || (p->BT > 0 && !dX)) return FLCE_ERR_INVALID_ARG;
  if (!aligned(loss, 4) || !aligned(dX, 16) || !aligned(dW, 16)) return FLCE_ERR_MISALIGNED;
  if (n_valid_global && !aligned(n_valid_global, 8)) return FLCE_ERR_MISALIGNED;
  Plan pl;
  make_plan(p, FLCE_OP_FUSED, &pl);
  if (ws_bytes < pl.total) return FLCE_ERR_WORKSPACE_TOO_SMALL;
  uint8_t* w = static_cast<uint8_t*>(ws);
  Ptrs q{X, W, labels, loss, reinterpret_cast<float*>(w + pl.off_lse), nullptr, dloss, dX, dW,
         w, n_valid_global};
  q.n_slices = n_slices;
  q.slice_done = reinterpret_cast<cudaEvent_t*>(const_cast<CUevent_st**>(slice_done));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if ((s = enqueue_shift(p, pl, &q, st)) != FLCE_OK) return s;
  if ((s = enqueue_labels(p, q, st)) != FLCE_OK) return s;
  if (pl.fused_fwd) return enqueue_fused_forward(p, pl, q, st);
  if ((s = enqueue_forward(p, pl, q, st)) != FLCE_OK) return s;
  if ((s = enqueue_backward(p, pl, q, st)) != FLCE_OK) return s;
  // the recompute schedule writes each vocabulary chunk's dW rows once, but
  // the slices are handed over together at the end
  return record_all_slices(q, st);
}

flce_status_t flce_fused(const flce_problem_t* p, const void* X, const void* W,
                         const int64_t* labels, float dloss, float* loss, void* dX, void* dW,
                         void* ws, size_t ws_bytes, struct CUstream_st* stream) {
  return fused_impl(p, X, W, labels, nullptr, dloss, loss, dX, dW, ws, ws_bytes, stream);
}

flce_status_t flce_fused_global(const flce_problem_t* p, const void* X, const void* W,
                                const int64_t* labels, const int64_t* n_valid_global,
                                float dloss, float* loss, void* dX, void* dW, void* ws,
                                size_t ws_bytes, struct CUstream_st* stream) {
  if (!n_valid_global) return FLCE_ERR_INVALID_ARG;
  return fused_impl(p, X, W, labels, n_valid_global, dloss, loss, dX, dW, ws, ws_bytes, stream);
}

flce_status_t flce_fused_global_sliced(const flce_problem_t* p, const void* X, const void* W,
                                       const int64_t* labels, const int64_t* n_valid_global,
                                       float dloss, float* loss, void* dX, void* dW, void* ws,
                                       size_t ws_bytes, int32_t n_slices,
                                       struct CUevent_st* const* slice_done,
                                       struct CUstream_st* stream) {
  if (n_slices < 1) return FLCE_ERR_INVALID_ARG;
  return fused_impl(p, X, W, labels, n_valid_global, dloss, loss, dX, dW, ws, ws_bytes, stream,
                    n_slices, slice_done);
}

int64_t flce_dw_slice_rows(int64_t V, int32_t n_slices) {
  if (V <= 0 || n_slices < 1 || n_slices > kMaxDwSlices) return 0;
  return dw_slice_rows(V, n_slices);
}

flce_status_t flce_count_valid(const flce_problem_t* p, const int64_t* labels, int64_t* n_valid,
                               struct CUstream_st* stream) {
  t_launches = 0;
  flce_status_t s = check_problem(p);
  if (s != FLCE_OK) return s;
  if (!n_valid || (p->BT > 0 && !labels)) return FLCE_ERR_INVALID_ARG;
  if (!aligned(n_valid, 8) || !aligned(labels, 8)) return FLCE_ERR_MISALIGNED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  prof_before(st);
  count_valid_kernel<<<1, 1024, 0, st>>>(labels, p->BT, p->shift_seq_len, p->ignore_index,
                                         n_valid);
  prof_after(st, K_COUNT_VALID);
  return cuda_status(cudaGetLastError());
}

flce_status_t flce_get_device_status(const void* ws, struct CUstream_st* stream,
                                     int32_t* device_status, int64_t* n_valid) {
  if (!ws) return FLCE_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  WsHeader h{};
  if (cudaStreamSynchronize(st) != cudaSuccess) return FLCE_ERR_CUDA;
  if (cudaMemcpy(&h, ws, sizeof h, cudaMemcpyDeviceToHost) != cudaSuccess) return FLCE_ERR_CUDA;
  if (device_status) *device_status = h.status;
  if (n_valid) *n_valid = h.n_valid;
  return FLCE_OK;
}

const char* flce_status_string(flce_status_t s) {
  switch (s) {
    case FLCE_OK: return "ok";
    case FLCE_ERR_INVALID_ARG: return "invalid argument";
    case FLCE_ERR_UNSUPPORTED: return "unsupported dtype or size";
    case FLCE_ERR_MISALIGNED: return "misaligned pointer or H not a multiple of 8";
    case FLCE_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case FLCE_ERR_LABEL_OUT_OF_RANGE: return "label outside [0, V) that is not ignore_index";
    case FLCE_ERR_TIMEOUT: return "a pipeline wait timed out";
    case FLCE_ERR_CUDA: return "CUDA error";
  }
  return "unknown status";
}

uint64_t flce_set_wait_limit_ns(uint64_t ns) {
  return g_wait_limit_ns.exchange(ns ? ns : 2000000000ull);
}

int32_t flce_last_launch_count(void) { return t_launches; }

flce_status_t flce_selftest_wait_timeout(void* ws, uint64_t limit_ns, struct CUstream_st* stream) {
  if (!ws || !aligned(ws, 256)) return FLCE_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  WsHeader* hdr = static_cast<WsHeader*>(ws);
  if (cudaMemsetAsync(hdr, 0, sizeof(WsHeader), st) != cudaSuccess) return FLCE_ERR_CUDA;
  selftest_wait_kernel<<<1, 32, 0, st>>>(hdr, limit_ns);
  return cuda_status(cudaGetLastError());
}

flce_status_t flce_selftest_approx(const float* x, int64_t n, float* out, struct CUstream_st* stream) {
  if (n < 0 || (n > 0 && (!x || !out))) return FLCE_ERR_INVALID_ARG;
  if (!aligned(x, 4) || !aligned(out, 4)) return FLCE_ERR_MISALIGNED;
  if (n == 0) return FLCE_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int blocks = int(cdiv(n, 256));
  if (blocks > 4096) blocks = 4096;
  approx_selftest_kernel<<<blocks, 256, 0, st>>>(x, n, out);
  return cuda_status(cudaGetLastError());
}

uint64_t flce_set_workspace_limit(uint64_t bytes) { return g_ws_limit.exchange(bytes); }

int32_t flce_set_schedule(int32_t schedule) {
  if (schedule < FLCE_SCHEDULE_AUTO || schedule > FLCE_SCHEDULE_FUSED_FORWARD) return -1;
  return g_schedule.exchange(schedule);
}

flce_status_t flce_profile_start(int32_t max_records) {
  std::lock_guard<std::mutex> lk(g_prof.mu);
  if (g_prof.on || max_records <= 0) return FLCE_ERR_INVALID_ARG;
  g_prof.ev = new cudaEvent_t[size_t(max_records) * 2]();
  g_prof.kind = new int32_t[size_t(max_records)]();
  for (int i = 0; i < 2 * max_records; ++i) {
    if (cudaEventCreate(&g_prof.ev[i]) != cudaSuccess) {
      for (int j = 0; j < i; ++j) cudaEventDestroy(g_prof.ev[j]);
      delete[] g_prof.ev;
      delete[] g_prof.kind;
      g_prof.ev = nullptr;
      g_prof.kind = nullptr;
      return FLCE_ERR_CUDA;
    }
  }
  g_prof.cap = max_records;
  g_prof.n = 0;
  g_prof.on = true;
  return FLCE_OK;
}

int32_t flce_profile_stop(float* ms, int32_t* kinds, int32_t max_out) {
  std::lock_guard<std::mutex> lk(g_prof.mu);
  if (!g_prof.on) return -1;
  const int n = g_prof.n;
  int out = 0;
  bool ok = n == 0 || cudaEventSynchronize(g_prof.ev[2 * n - 1]) == cudaSuccess;
  for (int i = 0; ok && i < n && i < max_out; ++i) {
    float t = 0.f;
    if (cudaEventElapsedTime(&t, g_prof.ev[2 * i], g_prof.ev[2 * i + 1]) != cudaSuccess) {
      ok = false;
      break;
    }
    if (ms) ms[i] = t;
    if (kinds) kinds[i] = g_prof.kind[i];
    ++out;
  }
  for (int i = 0; i < 2 * g_prof.cap; ++i) cudaEventDestroy(g_prof.ev[i]);
  delete[] g_prof.ev;
  delete[] g_prof.kind;
  g_prof.ev = nullptr;
  g_prof.kind = nullptr;
  g_prof.on = false;
  g_prof.cap = g_prof.n = 0;
  return ok ? out : -1;
}

// ------------------------ vocabulary parallelism ---------------------------

static flce_status_t vp_check(const flce_problem_t* p, int64_t v_offset, int64_t v_total) {
  flce_status_t s = check_problem(p);
  if (s != FLCE_OK) return s;
  if (p->shift_seq_len != 0) return FLCE_ERR_UNSUPPORTED;
  if (v_offset < 0 || v_total < v_offset + p->V) return FLCE_ERR_INVALID_ARG;
  if (v_total >= (int64_t(1) << 31)) return FLCE_ERR_UNSUPPORTED;
  return FLCE_OK;
}

flce_status_t flce_vp_forward(const flce_problem_t* p, int64_t v_offset, int64_t v_total,
                              const void* X, const void* W, const int64_t* labels, float* stats,
                              void* ws, size_t ws_bytes, struct CUstream_st* stream) {
  t_launches = 0;
  flce_status_t s = vp_check(p, v_offset, v_total);
  if (s != FLCE_OK) return s;
  if ((s = check_common(p, X, W, labels, ws)) != FLCE_OK) return s;
  if (p->BT > 0 && !stats) return FLCE_ERR_INVALID_ARG;
  if (!aligned(stats, 4)) return FLCE_ERR_MISALIGNED;
  Plan pl;
  make_plan(p, FLCE_OP_FORWARD, &pl);
  if (ws_bytes < pl.total) return FLCE_ERR_WORKSPACE_TOO_SMALL;
  pl.label_off = v_offset;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* w = static_cast<uint8_t*>(ws);
  WsHeader* hdr = reinterpret_cast<WsHeader*>(w);
  // the labels are global vocabulary ids: checked against the whole vocabulary
  prof_before(st);
  labels_kernel<<<1, 1024, 0, st>>>(labels, p->BT, v_total, p->ignore_index, hdr);
  prof_after(st, K_LABELS);
  FLCE_TRY(cudaGetLastError());
  const int64_t BT = pl.BT, V = pl.V, H = pl.H;
  if (BT == 0) return FLCE_OK;
  float2* partial = reinterpret_cast<float2*>(w + pl.off_partial);
  float* target = reinterpret_cast<float*>(w + pl.off_target);
  Ptrs q{X, W, labels, nullptr, nullptr, nullptr, 1.f, nullptr, nullptr, w};
  if (pl.tc) {
    CUtensorMap ma, mb;
    if (!make_map(&ma, X, H, BT, pl.ldx * 2, 64, kBM)) return FLCE_ERR_CUDA;
    if (!make_map(&mb, W, H, V, pl.ldw * 2, 64, b_box_rows())) return FLCE_ERR_CUDA;
    TcEpi ep = base_epi(p, pl, q);
    ep.partial = partial;
    ep.target = target;
    GemmArgs g{BT, V, H, true};
    g.wide_epi = pl.part_shift == 7;
    if (ep.softcap > 0.f)
      FLCE_TRY((launch_gemm<false, false, EPI_LSE_CAP>(ma, mb, ma, g, ep, device_sms(), st)));
    else
      FLCE_TRY((launch_gemm<false, false, EPI_LSE>(ma, mb, ma, g, ep, device_sms(), st)));
  } else {
    SimtEpi ep = base_simt(p, pl, q);
    ep.partial = partial;
    ep.target = target;
    prof_before(st);
    simt_logits_kernel<float, 0><<<dim3(unsigned(cdiv(V, 32)), unsigned(cdiv(BT, 32))),
                                   dim3(32, 8), 0, st>>>(static_cast<const float*>(X),
                                                         static_cast<const float*>(W), ep);
    prof_after(st, K_SIMT_LOGITS);
    FLCE_TRY(cudaGetLastError());
  }
  prof_before(st);
  vp_stats_kernel<<<unsigned(cdiv(BT, 256)), 256, 0, st>>>(
      partial, int(pl.part_tiles), BT, target, labels, p->ignore_index, v_offset, V, stats, hdr);
  prof_after(st, K_VP_STATS);
  return cuda_status(cudaGetLastError());
}

flce_status_t flce_vp_combine(const flce_problem_t* p, int32_t n_ranks, const float* stats_all,
                              const int64_t* labels, float* loss, float* lse, void* ws,
                              size_t ws_bytes, struct CUstream_st* stream) {
  t_launches = 0;
  flce_status_t s = vp_check(p, 0, p ? p->V : 0);
  if (s != FLCE_OK) return s;
  if (n_ranks < 1 || !loss || !ws || (p->BT > 0 && (!stats_all || !labels || !lse)))
    return FLCE_ERR_INVALID_ARG;
  if (!aligned(stats_all, 4) || !aligned(labels, 8) || !aligned(loss, 4) || !aligned(lse, 4) ||
      !aligned(ws, 256))
    return FLCE_ERR_MISALIGNED;
  // header and per-row losses, laid out as in the forward workspace
  const size_t off_rowloss = kHeaderBytes + align256(size_t(p->BT) * 4);
  if (ws_bytes < off_rowloss + align256(size_t(p->BT) * 4)) return FLCE_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* w = static_cast<uint8_t*>(ws);
  WsHeader* hdr = reinterpret_cast<WsHeader*>(w);
  float* rowloss = reinterpret_cast<float*>(w + off_rowloss);
  prof_before(st);
  labels_kernel<<<1, 1024, 0, st>>>(labels, p->BT, p->V, p->ignore_index, hdr);
  prof_after(st, K_LABELS);
  FLCE_TRY(cudaGetLastError());
  if (p->BT > 0) {
    prof_before(st);
    vp_combine_kernel<<<unsigned(cdiv(p->BT, 256)), 256, 0, st>>>(
        stats_all, n_ranks, p->BT, labels, p->ignore_index, lse, rowloss, hdr);
    prof_after(st, K_VP_COMBINE);
    FLCE_TRY(cudaGetLastError());
  }
  prof_before(st);
  finalize_kernel<<<1, 1024, 0, st>>>(rowloss, p->BT, hdr, loss);
  prof_after(st, K_FINALIZE);
  return cuda_status(cudaGetLastError());
}

flce_status_t flce_vp_backward(const flce_problem_t* p, int64_t v_offset, int64_t v_total,
                               const void* X, const void* W, const int64_t* labels,
                               const float* lse, const float* dloss, float* dX, void* dW,
                               void* ws, size_t ws_bytes, struct CUstream_st* stream) {
  t_launches = 0;
  flce_status_t s = vp_check(p, v_offset, v_total);
  if (s != FLCE_OK) return s;
  if ((s = check_common(p, X, W, labels, ws)) != FLCE_OK) return s;
  if (!dloss || !dW || (p->BT > 0 && (!lse || !dX))) return FLCE_ERR_INVALID_ARG;
  if (!aligned(dX, 16) || !aligned(dW, 16) || !aligned(lse, 4) || !aligned(dloss, 4))
    return FLCE_ERR_MISALIGNED;
  if ((eff_ld(p->lddx, p->H) * 4) % 16 != 0) return FLCE_ERR_MISALIGNED;
  Plan pl;
  const bool tc = p->dtype == FLCE_BF16;
  make_plan(p, tc ? kOpBackwardDxF32 : FLCE_OP_BACKWARD, &pl);
  if (ws_bytes < pl.total) return FLCE_ERR_WORKSPACE_TOO_SMALL;
  pl.dx_f32 = tc;
  pl.label_off = v_offset;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  Ptrs q{X, W, labels, nullptr, const_cast<float*>(lse), dloss, 1.f, dX, dW,
         static_cast<uint8_t*>(ws)};
  prof_before(st);
  labels_kernel<<<1, 1024, 0, st>>>(labels, p->BT, v_total, p->ignore_index,
                                    reinterpret_cast<WsHeader*>(ws));
  prof_after(st, K_LABELS);
  FLCE_TRY(cudaGetLastError());
  return enqueue_backward(p, pl, q, st);
}

size_t flce_vp_workspace_size(const flce_problem_t* p, int op) {
  if (check_problem(p) != FLCE_OK || p->shift_seq_len != 0) return 0;
  if (op != FLCE_OP_FORWARD && op != FLCE_OP_BACKWARD) return 0;
  Plan pl;
  make_plan(p, op == FLCE_OP_BACKWARD && p->dtype == FLCE_BF16 ? kOpBackwardDxF32 : op, &pl);
  return pl.total;
}

const char* flce_kernel_name(int32_t kind) {
  return (kind >= 0 && kind < K_NUM_KINDS) ? kKindNames[kind] : "unknown";
}

}  // extern "C"

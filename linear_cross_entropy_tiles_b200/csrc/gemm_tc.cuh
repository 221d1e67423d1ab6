// gemm_tc.cuh -- persistent, warp-specialised tcgen05 GEMM with the FLCE
// epilogues (the single-CTA kernel; gemm_tc2.cuh runs the same epilogues on
// CTA pairs).
//
// One CTA per SM, 192 threads:
//   warp 0      TMA producer: streams 128x64 A tiles and BNx64 B tiles (bf16,
//               128-byte swizzle) into a STAGES-deep shared-memory ring.
//   warp 1      allocates TMEM; lane 0 issues tcgen05.mma (M=128, N=BN, K=16)
//               into one of two fp32 accumulators (2*BN TMEM columns), so the
//               epilogue of tile t overlaps the main loop of tile t+1.
//   warps 2..5  epilogue: tcgen05.ld of 32 to 128 columns at a time, one
//               thread per accumulator row (TMEM lane), then one of
//     EPI_LSE  -- per-row online max / sum of exp over the tile's columns and
//                 the target-logit gather (the row max and row sum passes,
//                 steps 2 and 3 of PyTorch PR #126348's summary, done on the
//                 tile in registers instead of re-reading HBM);
//     EPI_GRAD -- G = (exp(y - lse) - onehot) * dy/dz * dloss / N, rounded to
//                 bf16 into the chunk buffer (the softmax recomputed from the
//                 saved row statistics, PR #126348 point b);
//     EPI_DX   -- dX tile: fp32 accumulate across vocabulary chunks, bf16 on
//                 the last chunk;
//     EPI_DW   -- dW tile: bf16 store;
//     EPI_LSE_Q -- EPI_LSE for the fused-in-forward schedule: also stores
//                 q = exp(y - R) * dy/dz (bf16) for every column against one
//                 reference R per row, with the (max, sum) partials; G is
//                 then diag(f) q up to one scalar and the label column.
// (_CAP variants apply the Gemma2 softcap.)
//
// Operands: A is M x K, B is N x K (D = A B^T).  Either may be K-major (rows
// of K contiguous) or MN-major (rows of M/N contiguous); MN-major tiles are
// loaded as 64-element-wide TMA boxes stacked along M/N.
//
// Every mbarrier wait is bounded in wall time.  A wait that gives up records
// FLCE_ERR_TIMEOUT in the status word, raises a shared abort flag that makes
// the other roles leave their loops, drains the copies and MMAs already in
// flight (again with a bound), frees TMEM and returns.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "sm100.cuh"

namespace flce {

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kTcThreads = 192;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.69314718055994531f;
constexpr int kStatusTimeout = 6;  // FLCE_ERR_TIMEOUT
// Bound on the drain waits of the abort path (copies and MMAs already issued
// finish in microseconds); independent of the user-set wait limit.
constexpr uint64_t kDrainLimitNs = 1000000000ull;

// EPI_DX is the generic "fp32 running sum across launches" epilogue: it also
// accumulates dW over row chunks in the fused-in-forward schedule.
// The *_CAP modes are the same epilogues with the logit softcap compiled in.
enum : int {
  EPI_LSE = 0, EPI_GRAD = 1, EPI_DX = 2, EPI_DW = 3, EPI_LSE_Q = 4,
  EPI_LSE_CAP = 5, EPI_GRAD_CAP = 6, EPI_LSE_Q_CAP = 7
};

struct TcShape {
  int M, N, K;              // this launch's GEMM: D[M x N] = A[M x K] B[N x K]^T
  int m_tiles, n_tiles, k_blocks, num_tiles;
  int m_fast;               // 1: consecutive tile ids walk along M first
  int a_mn_off, a_k_off;    // added to A's M and K coordinates
  int b_mn_off, b_k_off;    // added to B's N and K coordinates
  int k_splits;             // > 1: K is split; split s writes fp32 slab s (EPI_DX only)
};

struct TcEpi {
  int* status;              // device status word (0 = ok)
  unsigned long long wait_limit_ns;
  const int64_t* labels;    // [BT]
  int64_t ignore_index;
  int64_t BT, V, H;
  float softcap;            // > 0: y = softcap * tanh(z / softcap)
  // EPI_LSE
  float2* partial;          // [n_tiles][BT]: (max of y*log2e, sum of exp2(y*log2e - max))
  float* target;            // [BT]: y at the label column
  // EPI_GRAD
  const float* lse;         // [BT], natural log
  const float* dloss_dev;   // upstream gradient on the device, or null
  float dloss_host;         // used when dloss_dev is null
  const long long* n_valid; // device count of non-ignored rows
  __nv_bfloat16* G;         // chunk buffer, row stride ldg
  int64_t ldg;
  int64_t v0;               // vocabulary index of the chunk's first column / row
  // EPI_DX
  float* dx_acc;            // [BT][H] fp32 running sum over chunks, or the K-split slabs
  int64_t slab_stride;      // elements between K-split slabs
  __nv_bfloat16* dx;        // [BT][H]
  int dx_first, dx_last;
  // EPI_DW
  __nv_bfloat16* dw;        // [V][H]
  // Row strides (elements) of dx and dw where the epilogue stores them
  // itself rather than through a TMA map, and of the fp32 running sum dx_acc.
  int64_t ld_dx, ld_dw, ld_acc;
  // 1: the result is fp32 -- EPI_DW stores fp32 pieces (through an fp32 map,
  // or to dw32 without one); a running sum's last pass stores the fp32 sum
  // (to dx_acc, which then is the output) instead of converting it.
  int out_f32;
  float* dw32;
  // EPI_LSE_Q (fused-in-forward schedule): rows of this launch start at row0;
  // P is the chunk buffer [rows][ldp] of q = exp(y - R) dy/dz, bf16; ref, if
  // set, holds each chunk row's exponent reference R (log2 units), else R = 0
  int64_t row0;
  __nv_bfloat16* P;
  int64_t ldp;
  const float* ref;
  // Any mode: if set, a work unit runs only when one of the 32-row groups of
  // chunk rows its tile covers has a nonzero flag here (all roles skip the
  // others alike); for recomputing the few rows whose logits left the
  // shared reference's range.
  const int* row_group_flags;
  int n_groups;  // entries of row_group_flags
  // EPI_DX: the result is multiplied by row_scale[row] (chunk rows) when set,
  // and by dloss / N_valid (from n_valid, dloss_host) when scale_by_nvalid.
  const float* row_scale;
  int scale_by_nvalid;
  // EPI_LSE / EPI_GRAD: the vocabulary id of this launch's first W row (a
  // vocabulary-parallel rank's slice); labels are global ids.
  int64_t label_off;
  // bf16 output tiles stored by TMA: row added to the tile row (the
  // vocabulary offset of a dW chunk) and the output tensor's column count.
  int out_row_off;
  int out_cols;
  // EPI_DX running sums (one K split): 1 = store through the TMA sink, whose
  // map is then fp32 (the running sum) before the last pass and bf16 (the
  // result) on it.
  int tma_rmw;
};

// Where an epilogue's bf16 output chunks (32 columns of one row per thread)
// go.  Without a TMA sink they are stored to global memory directly; the
// CTA-pair kernel supplies one: each warp stages 32 rows x 64 columns in a
// 128-byte-swizzled shared-memory buffer (two per warp, used in turn) and
// stores the piece with one TMA instruction, so global writes are whole rows
// of 128 bytes instead of 16-byte fragments of 32 different rows.
struct TmaSink {
  const CUtensorMap* map;
  uint8_t* stage;     // this warp's nbuf 4 KB buffers (1024-byte aligned)
  int lane;
  int col0;           // tensor column of the tile's first column
  int row;            // tensor row of the warp's first row
  uint32_t* pieces;   // pieces this warp has stored so far (selects the buffer)
  int col_limit;      // the tensor's columns and rows: a piece that starts
  int row_limit;      // outside them is not stored (partial pieces are clipped)
  int nbuf;           // staging buffers of 4 KB (1 or 2)
};

__device__ __forceinline__ void put_bf16(TmaSink* tma, __nv_bfloat16* rowptr, int c,
                                         const uint32_t (&packed)[16]) {
  if (!tma) {
    if (rowptr) {
      uint4* dst = reinterpret_cast<uint4*>(rowptr + c * 32);
#pragma unroll
      for (int q = 0; q < 4; ++q)
        dst[q] = make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2],
                            packed[4 * q + 3]);
    }
    return;
  }
  uint8_t* buf = tma->stage + (tma->nbuf == 2 ? ((*tma->pieces & 1u) << 12) : 0u);
  if ((c & 1) == 0) {
    // The store that last read this buffer must be done with it: with two
    // buffers that is the one before the newest, with one the newest.
    if (tma->lane == 0) {
      if (tma->nbuf == 2)
        bulk_wait_group_read<1>();
      else
        bulk_wait_group_read<0>();
    }
    __syncwarp();
  }
  uint8_t* rowbuf = buf + tma->lane * 128;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int u = (c & 1) * 4 + q;  // 16-byte unit within the 128-byte row
    *reinterpret_cast<uint4*>(rowbuf + ((u ^ (tma->lane & 7)) << 4)) =
        make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
  }
  if (c & 1) {
    fence_proxy_async_smem();
    __syncwarp();
    const int col = tma->col0 + (c >> 1) * 64;
    // Warp-uniform.  Only a stored piece moves to the other buffer: the wait
    // above relies on the newest bulk group having read the other buffer.
    if (col < tma->col_limit && tma->row < tma->row_limit) {
      if (tma->lane == 0) {
        tma_store_2d(tma->map, buf, col, tma->row);
        bulk_commit_group();
      }
      ++*tma->pieces;
    }
  }
}

// One 32-column fp32 chunk (32 rows x 128 bytes, one 4 KB piece) through the
// sink: staged in a 128-byte-swizzled buffer and stored by one TMA
// instruction, like put_bf16's pieces of 64 bf16 columns.
__device__ __forceinline__ void put_f32(TmaSink* tma, int c, const float (&a)[32]) {
  uint8_t* buf = tma->stage + (tma->nbuf == 2 ? ((*tma->pieces & 1u) << 12) : 0u);
  if (tma->lane == 0) {
    if (tma->nbuf == 2)
      bulk_wait_group_read<1>();
    else
      bulk_wait_group_read<0>();
  }
  __syncwarp();
  uint8_t* rowbuf = buf + tma->lane * 128;
#pragma unroll
  for (int u = 0; u < 8; ++u)
    *reinterpret_cast<float4*>(rowbuf + ((u ^ (tma->lane & 7)) << 4)) =
        make_float4(a[4 * u], a[4 * u + 1], a[4 * u + 2], a[4 * u + 3]);
  fence_proxy_async_smem();
  __syncwarp();
  const int col = tma->col0 + c * 32;
  if (col < tma->col_limit && tma->row < tma->row_limit) {
    if (tma->lane == 0) {
      tma_store_2d(tma->map, buf, col, tma->row);
      bulk_commit_group();
    }
    ++*tma->pieces;
  }
}

__device__ __forceinline__ void tile_coords(const TcShape& sh, int t, int& mt, int& nt) {
  if (sh.m_fast) {
    mt = t % sh.m_tiles;
    nt = t / sh.m_tiles;
  } else {
    nt = t % sh.n_tiles;
    mt = t / sh.n_tiles;
  }
}

// Whether any of the launch's row groups is flagged (every thread of the CTA
// calls it once, in the prologue; true when no flags are given).
__device__ __forceinline__ bool any_group_flagged(const TcEpi& ep) {
  if (!ep.row_group_flags) return __syncthreads_or(1) != 0;
  int any = 0;
  for (int g = threadIdx.x; g < ep.n_groups; g += blockDim.x) any |= ep.row_group_flags[g];
  return __syncthreads_or(any) != 0;
}

// Whether the work unit whose output rows are [m_lo, m_lo + rows) of the
// launch runs: always, unless ep.row_group_flags asks for only the 32-row
// groups flagged there (none at all: `any` is false and nothing runs).
// Every role evaluates it for every unit alike.
__device__ __forceinline__ bool tile_wanted(const TcEpi& ep, const TcShape& sh, int m_lo,
                                            int rows, bool any = true) {
  if (!ep.row_group_flags) return true;
  if (!any) return false;
  const int g1 = min(m_lo + rows, sh.M);
  for (int g = m_lo; g < g1; g += 32)
    if (ep.row_group_flags[g >> 5]) return true;
  return false;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void record_timeout(const TcEpi& ep, volatile int* abort_flag) {
  *abort_flag = 1;
  atomicCAS(ep.status, 0, kStatusTimeout);
}

// ------------------------------- epilogues ---------------------------------
// Every epilogue walks the thread's row of the tile in groups of kLoadCols
// columns: one tcgen05.ld of the whole group and one wait, then the group is
// processed from registers in 32-column chunks (chunk index c, values v[32]).
// Group width per epilogue: 128 columns where the per-element work is a
// conversion or an add (dX, dW), 32 where it is the exponential arithmetic
// (LSE, q, G), which schedules better on short groups (both measured).
__device__ __forceinline__ void tmem_ld_group(uint32_t taddr, uint32_t (&r)[128]) {
  tmem_ld_32x32b_x128(taddr, r);
}
__device__ __forceinline__ void tmem_ld_group(uint32_t taddr, uint32_t (&r)[32]) {
  tmem_ld_32x32b_x32(taddr, r);
}
__device__ __forceinline__ void tmem_ld_group(uint32_t taddr, uint32_t (&r)[64]) {
  tmem_ld_32x32b_x32(taddr, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
  tmem_ld_32x32b_x32(taddr + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
}

// 2^x on the SFU (ex2.approx.ftz: relative error ~2^-22; inputs here are
// <= 0 up to rounding, results below 2^-126 flush to 0).
__device__ __forceinline__ float ex2a(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// tanh(x) = 1 - 2 / (e^(2x) + 1), with e^(2x) = 2^(2 x log2 e) on the SFU.
// Absolute error ~1e-7 over the whole range (saturates to +-1 exactly).
__device__ __forceinline__ float tanh_fast(float x) {
  return 1.f - __fdividef(2.f, ex2a(x * (2.f * kLog2e)) + 1.f);
}

// The softcap y = c tanh(z / c) and its derivative 1 - tanh^2(z / c).
template <bool CAP>
__device__ __forceinline__ float capped(float z, float sc, float inv_sc, float* d) {
  if (!CAP) {
    *d = 1.f;
    return z;
  }
  const float t = tanh_fast(z * inv_sc);
  *d = 1.f - t * t;
  return sc * t;
}

// v[idx] for a per-thread idx in [0, 32), as a five-level select tree
// (registers cannot be indexed by a per-thread value).
__device__ __forceinline__ float pick32(const uint32_t* v, int idx) {
  float a[16], b[8], c[4], d[2];
#pragma unroll
  for (int k = 0; k < 16; ++k) a[k] = __uint_as_float((idx & 16) ? v[k + 16] : v[k]);
#pragma unroll
  for (int k = 0; k < 8; ++k) b[k] = (idx & 8) ? a[k + 8] : a[k];
#pragma unroll
  for (int k = 0; k < 4; ++k) c[k] = (idx & 4) ? b[k + 4] : b[k];
#pragma unroll
  for (int k = 0; k < 2; ++k) d[k] = (idx & 2) ? c[k + 2] : c[k];
  return (idx & 1) ? d[1] : d[0];
}

// Whether any thread of the warp has its label in columns [c0, c0 + 32) of
// the tile, and whether this one does.
__device__ __forceinline__ bool label_in_chunk(int lab_col, int c0, bool* mine) {
  *mine = lab_col >= c0 && lab_col < c0 + 32;
  return __any_sync(0xffffffffu, *mine);
}

// Epilogues process chunks [c_lo, c_hi) of 32 columns of the 256-column
// tile; `part` is the index of the LSE partial those columns form.
template <int BN, bool CAP>
__device__ __forceinline__ void epi_lse(const TcEpi& ep, const TcShape& sh, int m0, int n0,
                                        int part, int r, uint32_t taddr, int c_lo = 0,
                                        int c_hi = BN / 32) {
  const int64_t row = int64_t(m0) + r;
  const bool row_ok = row < sh.M;
  const int64_t lab = row_ok ? __ldg(ep.labels + row) : ep.ignore_index;
  const int64_t labl = lab - ep.label_off;  // the label's column in this launch's W rows
  const int lab_col = (lab != ep.ignore_index && labl >= n0 && labl < int64_t(n0) + BN)
                          ? int(labl - n0) : -1;
  const float sc = ep.softcap;
  const float inv_sc = CAP ? 1.f / ep.softcap : 0.f;
  const int ncols = sh.N - n0;  // tile columns inside the vocabulary
  const bool full = ncols >= c_hi * 32;
  float m = -INFINITY, s = 0.f, tgt = 0.f;
#pragma unroll 1
  for (int c = c_lo; c < c_hi; ++c) {
    uint32_t v[32];
    tmem_ld_32x32b_x32(taddr + c * 32, v);
    tmem_ld_wait();
    bool mine;
    if (label_in_chunk(lab_col, c * 32, &mine) && mine) {
      float d;
      tgt = capped<CAP>(pick32(v, lab_col - c * 32), sc, inv_sc, &d);
    }
    // the chunk's max of y: the softcap is increasing, so cap the max of z
    float zmax = -INFINITY;
#pragma unroll
    for (int k = 0; k < 32; ++k)
      if (full || c * 32 + k < ncols) zmax = fmaxf(zmax, __uint_as_float(v[k]));
    float dd;
    const float mn = fmaxf(m, capped<CAP>(zmax, sc, inv_sc, &dd) * kLog2e);
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
    for (int k = 0; k < 32; k += 4) {
      float p[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float d;
        const float y = capped<CAP>(__uint_as_float(v[k + e]), sc, inv_sc, &d);
        p[e] = ex2a(fmaf(y, kLog2e, -mn));
        if (!full && c * 32 + k + e >= ncols) p[e] = 0.f;
      }
      a0 += p[0];
      a1 += p[1];
      a2 += p[2];
      a3 += p[3];
    }
    s = s * ex2a(m - mn) + ((a0 + a1) + (a2 + a3));
    m = mn;
  }
  // Columns wholly past the vocabulary form no partial (the partial array
  // has one slice per chunk range that starts inside it).
  if (row_ok && ncols > c_lo * 32) {
    ep.partial[size_t(part) * size_t(ep.BT) + size_t(row)] = make_float2(m, s);
    if (lab_col >= c_lo * 32 && lab_col < c_hi * 32) ep.target[row] = tgt;
  }
}

template <int BN, bool CAP>
__device__ __forceinline__ void epi_grad(const TcEpi& ep, const TcShape& sh, int m0, int n0,
                                         int r, uint32_t taddr, TmaSink* tma = nullptr,
                                         int c_lo = 0, int c_hi = BN / 32) {
  const int64_t row = int64_t(m0) + r;
  const bool row_ok = row < sh.M;
  const int64_t lab = row_ok ? __ldg(ep.labels + row) : ep.ignore_index;
  const bool valid = row_ok && lab != ep.ignore_index;
  const long long nv = *ep.n_valid;
  const float dl = ep.dloss_dev ? *ep.dloss_dev : ep.dloss_host;
  const float scale = (valid && nv > 0) ? dl / float(nv) : 0.f;
  // An ignored row gets lse = +inf, so every exp is 0 and G is 0 exactly.
  const float lse2 = (valid && nv > 0) ? __ldg(ep.lse + row) * kLog2e : INFINITY;
  const int64_t vbase = ep.v0 + n0;  // vocabulary index of tile column 0
  const int64_t labl = lab - ep.label_off;
  const int lab_col = (valid && labl >= vbase && labl < vbase + BN) ? int(labl - vbase) : -1;
  const int64_t vlim = ep.V - vbase;  // tile columns >= vlim are padding
  const bool full = vlim >= c_hi * 32;
  const float sc = ep.softcap;
  const float inv_sc = CAP ? 1.f / ep.softcap : 0.f;
  __nv_bfloat16* gout = ep.G + row * ep.ldg + n0;
#pragma unroll 1
  for (int c = c_lo; c < c_hi; ++c) {
    uint32_t v[32];
    tmem_ld_32x32b_x32(taddr + c * 32, v);
    tmem_ld_wait();
    float g[32];
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      float d;
      const float y = capped<CAP>(__uint_as_float(v[k]), sc, inv_sc, &d);
      g[k] = ex2a(fmaf(y, kLog2e, -lse2)) * (CAP ? d * scale : scale);
      if (!full && c * 32 + k >= vlim) g[k] = 0.f;
    }
    bool mine;
    if (label_in_chunk(lab_col, c * 32, &mine)) {
      // the label column: (p - 1) * dy/dz * scale
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        if (mine && c * 32 + k == lab_col) {
          float d;
          const float y = capped<CAP>(__uint_as_float(v[k]), sc, inv_sc, &d);
          g[k] = (ex2a(fmaf(y, kLog2e, -lse2)) - 1.f) * d * scale;
        }
      }
    }
    uint32_t packed[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) packed[k] = pack_bf16x2(g[2 * k], g[2 * k + 1]);
    put_bf16(tma, row_ok ? gout : nullptr, c, packed);
  }
}

// LC: columns fetched from TMEM per wait (fewer when registers are scarce).
template <int BN, int LC = 128>
__device__ __forceinline__ void epi_dx(const TcEpi& ep, const TcShape& sh, int m0, int n0,
                                       int r, uint32_t taddr, int split = 0,
                                       TmaSink* tma = nullptr, int c_lo = 0,
                                       int c_hi = BN / 32) {
  constexpr int kLoadCols = LC;
  const int64_t row = int64_t(m0) + r;
  const bool row_ok = row < sh.M;
  // A single pass over K: the tile is the result; bf16 out through the sink.
  const bool direct = tma && sh.k_splits == 1 && ep.dx_first && ep.dx_last;
  // K-split partial: fp32 into this split's slab; a reduction kernel sums them.
  float* slab = ep.dx_acc + int64_t(split) * ep.slab_stride + row * ep.H;
  // Otherwise a running sum in fp32 (streamed: read and written once per launch).
  float* accrow = ep.dx_acc + row * ep.ld_acc;
  // The tile's factor (1 unless the launch asks for a row or global scale);
  // K-split slabs stay unscaled, their reduction applies it.
  float fac = 1.f;
  if (ep.row_scale) fac = row_ok ? ep.row_scale[row] : 0.f;
  if (ep.scale_by_nvalid) {
    const long long nv = *ep.n_valid;
    fac *= nv > 0 ? ep.dloss_host / float(nv) : 0.f;
  }
#pragma unroll 1
  for (int gq = c_lo * 32 / kLoadCols; gq < c_hi * 32 / kLoadCols; ++gq) {
    uint32_t vg[kLoadCols];
    tmem_ld_group(taddr + gq * kLoadCols, vg);
    tmem_ld_wait();
#pragma unroll
    for (int cc = 0; cc < kLoadCols / 32; ++cc) {
      const int c = gq * (kLoadCols / 32) + cc;
      const uint32_t* v = vg + cc * 32;
      if (direct) {
        if (ep.out_f32) {
          float a[32];
#pragma unroll
          for (int k = 0; k < 32; ++k) a[k] = __uint_as_float(v[k]) * fac;
          put_f32(tma, c, a);
          continue;
        }
        uint32_t packed[16];
#pragma unroll
        for (int k = 0; k < 16; ++k)
          packed[k] = pack_bf16x2(__uint_as_float(v[2 * k]) * fac,
                                  __uint_as_float(v[2 * k + 1]) * fac);
        put_bf16(tma, nullptr, c, packed);
        continue;
      }
      if (tma && ep.tma_rmw && sh.k_splits == 1) {
        // Running sum through the sink: every lane takes part in the staged
        // store (whole 128-byte rows; rows and columns past the tensor are
        // clipped by the TMA store, and their sum is never read).
        const int64_t c0 = int64_t(n0) + c * 32;
        float a[32];
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          float4 pv = make_float4(0.f, 0.f, 0.f, 0.f);
          if (row_ok && !ep.dx_first && c0 + 4 * g < ep.H)
            pv = __ldcs(reinterpret_cast<const float4*>(accrow + c0 + 4 * g));
          a[4 * g] = fmaf(__uint_as_float(v[4 * g]), fac, pv.x);
          a[4 * g + 1] = fmaf(__uint_as_float(v[4 * g + 1]), fac, pv.y);
          a[4 * g + 2] = fmaf(__uint_as_float(v[4 * g + 2]), fac, pv.z);
          a[4 * g + 3] = fmaf(__uint_as_float(v[4 * g + 3]), fac, pv.w);
        }
        if (!ep.dx_last || ep.out_f32) {
          put_f32(tma, c, a);
        } else {
          uint32_t packed[16];
#pragma unroll
          for (int k = 0; k < 16; ++k) packed[k] = pack_bf16x2(a[2 * k], a[2 * k + 1]);
          put_bf16(tma, nullptr, c, packed);
        }
        continue;
      }
      if (!row_ok) continue;
      const int64_t col0 = int64_t(n0) + c * 32;
      if (sh.k_splits > 1) {
#pragma unroll
        for (int g8 = 0; g8 < 4; ++g8) {
          const int64_t col = col0 + g8 * 8;
          if (col >= ep.H) break;
          const uint32_t* u = v + g8 * 8;
          *reinterpret_cast<uint4*>(slab + col) = make_uint4(u[0], u[1], u[2], u[3]);
          *reinterpret_cast<uint4*>(slab + col + 4) = make_uint4(u[4], u[5], u[6], u[7]);
        }
        continue;
      }
      float4 prev[8];
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        prev[g] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (!ep.dx_first && col0 + 4 * g < ep.H)
          prev[g] = __ldcs(reinterpret_cast<const float4*>(accrow + col0 + 4 * g));
      }
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        const int64_t col = col0 + 4 * g;
        if (col >= ep.H) break;
        const float4 a = make_float4(fmaf(__uint_as_float(v[4 * g]), fac, prev[g].x),
                                     fmaf(__uint_as_float(v[4 * g + 1]), fac, prev[g].y),
                                     fmaf(__uint_as_float(v[4 * g + 2]), fac, prev[g].z),
                                     fmaf(__uint_as_float(v[4 * g + 3]), fac, prev[g].w));
        if (!ep.dx_last || ep.out_f32) {
          __stcs(reinterpret_cast<float4*>(accrow + col), a);
        } else {
          *reinterpret_cast<uint2*>(ep.dx + row * ep.ld_dx + col) =
              make_uint2(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w));
        }
      }
    }
  }
}

template <int BN>
__device__ __forceinline__ void epi_dw(const TcEpi& ep, const TcShape& sh, int m0, int n0,
                                       int r, uint32_t taddr, TmaSink* tma = nullptr,
                                       int c_lo = 0, int c_hi = BN / 32) {
  constexpr int kLoadCols = 128;
  const int64_t lrow = int64_t(m0) + r;  // row within the chunk
  const int64_t vrow = ep.v0 + lrow;     // vocabulary row of dW
  const bool row_ok = lrow < sh.M && vrow < ep.V;
#pragma unroll 1
  for (int gq = c_lo * 32 / kLoadCols; gq < c_hi * 32 / kLoadCols; ++gq) {
    uint32_t vg[kLoadCols];
    tmem_ld_group(taddr + gq * kLoadCols, vg);
    tmem_ld_wait();
#pragma unroll
    for (int cc = 0; cc < kLoadCols / 32; ++cc) {
      const int c = gq * (kLoadCols / 32) + cc;
      const uint32_t* v = vg + cc * 32;
      if (tma) {
        if (ep.out_f32) {
          float a[32];
#pragma unroll
          for (int k = 0; k < 32; ++k) a[k] = __uint_as_float(v[k]);
          put_f32(tma, c, a);
          continue;
        }
        uint32_t packed[16];
#pragma unroll
        for (int k = 0; k < 16; ++k)
          packed[k] = pack_bf16x2(__uint_as_float(v[2 * k]), __uint_as_float(v[2 * k + 1]));
        put_bf16(tma, nullptr, c, packed);
        continue;
      }
      if (!row_ok) continue;
#pragma unroll
      for (int g8 = 0; g8 < 4; ++g8) {
        const int64_t col = int64_t(n0) + c * 32 + g8 * 8;
        if (col >= ep.H) break;
        const uint32_t* u = v + g8 * 8;
        if (ep.out_f32) {
          float* d = ep.dw32 + vrow * ep.ld_dw + col;
          *reinterpret_cast<uint4*>(d) = make_uint4(u[0], u[1], u[2], u[3]);
          *reinterpret_cast<uint4*>(d + 4) = make_uint4(u[4], u[5], u[6], u[7]);
          continue;
        }
        *reinterpret_cast<uint4*>(ep.dw + vrow * ep.ld_dw + col) = make_uint4(
            pack_bf16x2(__uint_as_float(u[0]), __uint_as_float(u[1])),
            pack_bf16x2(__uint_as_float(u[2]), __uint_as_float(u[3])),
            pack_bf16x2(__uint_as_float(u[4]), __uint_as_float(u[5])),
            pack_bf16x2(__uint_as_float(u[6]), __uint_as_float(u[7])));
      }
    }
  }
}

// One 32-column chunk of the fused-in-forward epilogue: for each column
// q = exp2(y log2(e) - R) * dy/dz as bf16 through the sink (0 for a row whose
// label is ignored), the running maximum of y and sum of exp2(y log2(e) - R),
// and y at the label column if it lies here.  MASK: some
// columns lie past the vocabulary (ncols); full ranges compile without the
// per-column test.
template <bool CAP, bool MASK>
__device__ __forceinline__ void lse_q_chunk(const uint32_t (&cur)[32], int c, float R, float sc,
                                            float inv_sc, int lab_col, bool keep, int ncols,
                                            TmaSink* tma, __nv_bfloat16* prow, float (&a)[4],
                                            float& mx, float& tgt) {
  bool mine;
  if (label_in_chunk(lab_col, c * 32, &mine) && mine) {
    float d;
    tgt = capped<CAP>(pick32(cur, lab_col - c * 32), sc, inv_sc, &d);
  }
  uint32_t packed[16];
#pragma unroll
  for (int k = 0; k < 32; k += 2) {
    float pv[2], qv[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float d;
      const float y = capped<CAP>(__uint_as_float(cur[k + e]), sc, inv_sc, &d);
      const bool in = !MASK || c * 32 + k + e < ncols;
      mx = in ? fmaxf(mx, y) : mx;  // in y; the caller scales it by log2(e)
      pv[e] = in ? ex2a(fmaf(y, kLog2e, -R)) : 0.f;
      qv[e] = keep ? (CAP ? pv[e] * d : pv[e]) : 0.f;
    }
    a[(k & 2) + 0] += pv[0];
    a[(k & 2) + 1] += pv[1];
    packed[k / 2] = pack_bf16x2(qv[0], qv[1]);
  }
  put_bf16(tma, prow, c, packed);
}

// One pass over a warp's columns [c_lo, c_lo + NCH) of the tile, two chunks
// per iteration so the TMEM load of the next chunk is in flight while the
// current one is processed.
template <bool CAP, bool MASK, int NCH>
__device__ __forceinline__ void epi_lse_q_range(const TcEpi& ep, float R, bool keep, int lab_col,
                                                int ncols, uint32_t taddr, TmaSink* tma,
                                                __nv_bfloat16* prow, int c_lo, float* m_out,
                                                float* s_out, float* tgt_out) {
  static_assert(NCH % 2 == 0, "chunks are handled in pairs");
  const float sc = ep.softcap;
  const float inv_sc = CAP ? 1.f / ep.softcap : 0.f;
  float a[4] = {0.f, 0.f, 0.f, 0.f};  // four running sums: fixed order, short chains
  float mx = -INFINITY, tgt = 0.f;
  uint32_t v0[32], v1[32];
  tmem_ld_32x32b_x32(taddr + c_lo * 32, v0);
  tmem_ld_wait_regs(v0);
#pragma unroll 1
  for (int i = 0; i < NCH; i += 2) {
    const int c = c_lo + i;
    tmem_ld_32x32b_x32(taddr + (c + 1) * 32, v1);
    lse_q_chunk<CAP, MASK>(v0, c, R, sc, inv_sc, lab_col, keep, ncols, tma, prow, a, mx, tgt);
    __syncwarp();
    tmem_ld_wait_regs(v1);
    const bool more = i + 2 < NCH;
    if (more) tmem_ld_32x32b_x32(taddr + (c + 2) * 32, v0);
    lse_q_chunk<CAP, MASK>(v1, c + 1, R, sc, inv_sc, lab_col, keep, ncols, tma, prow, a, mx,
                           tgt);
    if (more) {
      __syncwarp();
      tmem_ld_wait_regs(v0);
    }
  }
  *m_out = mx * kLog2e;  // largest y, in log2 units
  *s_out = (a[0] + a[1]) + (a[2] + a[3]);
  *tgt_out = tgt;
}

// Fused-in-forward epilogue.  Every row of the chunk shares one exponent
// reference R (log2 units) across all its vocabulary tiles -- 0, or for a
// row being recomputed because its logits left [-64, 64] (see lse_q_kernel)
// the row's exact maximum from ep.ref -- so that G = (dloss / N) diag(f) Q
// with one factor f_i = exp2(R_i - lse_i log2 e) per row, which the dX
// epilogue and the prescaled X of the dW GEMM apply: the chunk buffer is
// never rewritten.  Stores q = exp2(y log2 e - R) * dy/dz (bf16) for every
// column, zeros for ignored rows, and per (slice, row) the partial (largest
// y log2 e, sum of exp2(y log2 e - R)) plus the label's y.
// The label of the row this thread drains in the tile starting at chunk row
// m0, loaded before the accumulator is ready (its latency then hides behind
// the wait); ignore_index past the chunk.
__device__ __forceinline__ int64_t epi_row_label(const TcEpi& ep, const TcShape& sh, int m0,
                                                 int r) {
  const int64_t lrow = int64_t(m0) + r;
  return lrow < sh.M ? __ldg(ep.labels + ep.row0 + lrow) : ep.ignore_index;
}

template <int BN, bool CAP, int NCH = BN / 32>
__device__ __forceinline__ void epi_lse_q(const TcEpi& ep, const TcShape& sh, int m0, int n0,
                                          int part, int r, uint32_t taddr,
                                          TmaSink* tma = nullptr, int c_lo = 0,
                                          int c_hi = BN / 32, int64_t lab_pre = INT64_MIN) {
  const int64_t lrow = int64_t(m0) + r;  // row within the chunk
  // A recomputation touches only the flagged 32-row groups: exactly this
  // warp's rows (warp-uniform), so the rows of other groups keep what the
  // first pass and its finishing kernel wrote.
  if (ep.row_group_flags && ep.row_group_flags[lrow >> 5] == 0) return;
  const int64_t row = ep.row0 + lrow;    // row of X
  const bool row_ok = lrow < sh.M;
  const int64_t lab = lab_pre != INT64_MIN ? lab_pre : epi_row_label(ep, sh, m0, r);
  const bool keep = lab != ep.ignore_index;
  const int lab_col = (keep && lab >= n0 && lab < int64_t(n0) + BN) ? int(lab - n0) : -1;
  const int ncols = sh.N - n0;  // columns of this tile inside the vocabulary
  const float R = (ep.ref && row_ok) ? ep.ref[lrow] : 0.f;
  __nv_bfloat16* prow = row_ok ? ep.P + lrow * ep.ldp + n0 : nullptr;
  float m, s, tgt;
  if (ncols >= c_hi * 32)
    epi_lse_q_range<CAP, false, NCH>(ep, R, keep, lab_col, ncols, taddr, tma, prow, c_lo, &m,
                                     &s, &tgt);
  else
    epi_lse_q_range<CAP, true, NCH>(ep, R, keep, lab_col, ncols, taddr, tma, prow, c_lo, &m, &s,
                                    &tgt);
  // Columns wholly past the vocabulary form no partial.
  if (row_ok && ncols > c_lo * 32) {
    ep.partial[size_t(part) * size_t(ep.BT) + size_t(row)] = make_float2(m, s);
    if (lab_col >= c_lo * 32 && lab_col < c_hi * 32) ep.target[row] = tgt;
  }
}

// ------------------------------- the kernel --------------------------------

template <int BN, int STAGES>
struct TcSmem {
  static constexpr uint32_t kABytes = kBM * kBK * 2;
  static constexpr uint32_t kBBytes = BN * kBK * 2;
  static constexpr uint32_t kStageBytes = kABytes + kBBytes;
  static constexpr uint32_t kBarrierBytes = 256;
  // 1024 bytes of slack to align the ring to the 128B-swizzle atom.
  static constexpr uint32_t kTotal = STAGES * kStageBytes + kBarrierBytes + 1024;
  static constexpr uint32_t kTmemCols = (2 * BN <= 32) ? 32 : (2 * BN <= 64) ? 64
                                        : (2 * BN <= 128) ? 128 : (2 * BN <= 256) ? 256 : 512;
};

template <int BN, bool A_MN, bool B_MN, int MODE, int STAGES>
__global__ void __launch_bounds__(kTcThreads, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                   const __grid_constant__ CUtensorMap tmB, const TcShape sh, const TcEpi ep) {
  using L = TcSmem<BN, STAGES>;
  static_assert(BN % 64 == 0 && BN >= 64 && BN <= 256, "BN must be 64..256, multiple of 64");
  constexpr uint32_t kIdesc = make_idesc_bf16(kBM, BN, A_MN, B_MN);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * L::kStageBytes);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 128);
    }
    mbar_init(drain, 1);
    *abort_flag = (*reinterpret_cast<volatile int*>(ep.status) != 0) ? 2 : 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const bool any = any_group_flagged(ep);  // a recomputation with nothing flagged: no units
  const bool skip = *abort_flag != 0 || !any;  // (or an earlier kernel of this call failed)
  const uint64_t limit = ep.wait_limit_ns;

  if (!skip && warp == 0 && lane == 0) {
    // ------------------------------ producer ------------------------------
    const uint64_t pol_a = policy_evict_normal();
    const uint64_t pol_b = policy_evict_normal();
    uint32_t s = 0, ph = 0;
    uint32_t armed = 0;  // stages armed at least once
    uint32_t armed_ph[STAGES];
#pragma unroll
    for (int i = 0; i < STAGES; ++i) armed_ph[i] = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < sh.num_tiles; t += gridDim.x) {
      int mt, nt;
      tile_coords(sh, t, mt, nt);
      if (!tile_wanted(ep, sh, mt * kBM, kBM)) continue;
      const int m0 = mt * kBM + sh.a_mn_off;
      const int n0 = nt * BN + sh.b_mn_off;
      for (int kb = 0; kb < sh.k_blocks; ++kb) {
        if (!mbar_wait_bounded(&empty[s], ph ^ 1u, limit, abort_flag)) {
          record_timeout(ep, abort_flag);
          ok = false;
          break;
        }
        uint8_t* sa = smem + s * L::kStageBytes;
        uint8_t* sb = sa + L::kABytes;
        mbar_arrive_expect_tx(&full[s], L::kStageBytes);
        armed |= 1u << s;
        armed_ph[s] = ph;
        const int ka = kb * kBK + sh.a_k_off;
        const int kbb = kb * kBK + sh.b_k_off;
        if (!A_MN) {
          tma_load_2d(sa, &tmA, &full[s], ka, m0, pol_a);
        } else {
          tma_load_2d(sa, &tmA, &full[s], m0, ka, pol_a);
          tma_load_2d(sa + 8192, &tmA, &full[s], m0 + 64, ka, pol_a);
        }
        if (!B_MN) {
          tma_load_2d(sb, &tmB, &full[s], kbb, n0, pol_b);
        } else {
#pragma unroll
          for (int j = 0; j < BN / 64; ++j)
            tma_load_2d(sb + j * 8192, &tmB, &full[s], n0 + 64 * j, kbb, pol_b);
        }
        if (++s == STAGES) {
          s = 0;
          ph ^= 1u;
        }
      }
    }
    if (!ok || *abort_flag) {
      // Let every copy already issued land before the CTA's shared memory goes away.
      for (int i = 0; i < STAGES; ++i)
        if (armed & (1u << i)) mbar_wait_bounded(&full[i], armed_ph[i], kDrainLimitNs, nullptr);
    }
  } else if (!skip && warp == 1 && lane == 0) {
    // ------------------------------ MMA issuer -----------------------------
    uint32_t s = 0, ph = 0, acc = 0, aph = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < sh.num_tiles; t += gridDim.x) {
      {
        int mt, nt;
        tile_coords(sh, t, mt, nt);
        if (!tile_wanted(ep, sh, mt * kBM, kBM)) continue;
      }
      if (!mbar_wait_bounded(&tempty[acc], aph ^ 1u, limit, abort_flag)) {
        record_timeout(ep, abort_flag);
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t d = tmem_base + acc * BN;
      for (int kb = 0; kb < sh.k_blocks; ++kb) {
        if (!mbar_wait_bounded(&full[s], ph, limit, abort_flag)) {
          record_timeout(ep, abort_flag);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_addr = smem_u32(smem + s * L::kStageBytes);
        const uint32_t b_addr = a_addr + L::kABytes;
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk) {
          const uint64_t ad = A_MN ? make_sdesc_sw128(a_addr + kk * 2048, 8192, 1024)
                                   : make_sdesc_sw128(a_addr + kk * 32, 16, 1024);
          const uint64_t bd = B_MN ? make_sdesc_sw128(b_addr + kk * 2048, 8192, 1024)
                                   : make_sdesc_sw128(b_addr + kk * 32, 16, 1024);
          umma_bf16(d, ad, bd, kIdesc, (kb | kk) != 0 ? 1u : 0u);
        }
        umma_commit(&empty[s]);
        if (++s == STAGES) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (!ok) break;
      umma_commit(&tfull[acc]);
      acc ^= 1u;
      if (acc == 0) aph ^= 1u;
    }
    // Wait until every MMA issued above has finished with TMEM and smem.
    umma_commit(drain);
    mbar_wait_bounded(drain, 0, kDrainLimitNs, nullptr);
  } else if (!skip && warp >= 2) {
    // ------------------------------- epilogue ------------------------------
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int r = q * 32 + lane;
    uint32_t acc = 0, aph = 0;
    for (int t = blockIdx.x; t < sh.num_tiles; t += gridDim.x) {
      int mt, nt;
      tile_coords(sh, t, mt, nt);
      if (!tile_wanted(ep, sh, mt * kBM, kBM)) continue;
      // Every lane polls; all must agree before the warp-wide tcgen05.ld.
      const bool got = mbar_wait_bounded(&tfull[acc], aph, limit, abort_flag);
      if (!__all_sync(0xffffffffu, got)) {
        if (lane == 0) record_timeout(ep, abort_flag);
        break;
      }
      tc_fence_after();
      const uint32_t taddr = tmem_base + (uint32_t(q * 32) << 16) + acc * BN;
      const int m0 = mt * kBM;
      const int n0 = nt * BN;
      if (MODE == EPI_LSE) epi_lse<BN, false>(ep, sh, m0, n0, nt, r, taddr);
      if (MODE == EPI_LSE_CAP) epi_lse<BN, true>(ep, sh, m0, n0, nt, r, taddr);
      if (MODE == EPI_GRAD) epi_grad<BN, false>(ep, sh, m0, n0, r, taddr);
      if (MODE == EPI_GRAD_CAP) epi_grad<BN, true>(ep, sh, m0, n0, r, taddr);
      if (MODE == EPI_DX) epi_dx<BN>(ep, sh, m0, n0, r, taddr);
      if (MODE == EPI_DW) epi_dw<BN>(ep, sh, m0, n0, r, taddr);
      if (MODE == EPI_LSE_Q) epi_lse_q<BN, false>(ep, sh, m0, n0, nt, r, taddr);
      if (MODE == EPI_LSE_Q_CAP) epi_lse_q<BN, true>(ep, sh, m0, n0, nt, r, taddr);
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
      acc ^= 1u;
      if (acc == 0) aph ^= 1u;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, L::kTmemCols);
  }
}

}  // namespace flce

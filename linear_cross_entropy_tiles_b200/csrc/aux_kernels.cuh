// aux_kernels.cuh -- the small integer / reduction steps of FLCE and the
// CUDA-core (SIMT) path used for fp32 inputs.
//
//   labels_kernel    count N_valid (labels != ignore_index) and flag labels
//                    outside [0, V); resets the call's status word.
//   combine_kernel   fold the per-(tile, row) partial (max, sum-exp) pairs of
//                    the forward GEMM into lse_i in a fixed tile order, and
//                    the per-row NLL lse_i - y_i,label.
//   finalize_kernel  loss = sum of per-row NLL over valid rows / N_valid,
//                    summed in a fixed order in fp64 (0 when N_valid = 0).
//   simt_*           fp32 tiles on CUDA cores for the same steps; fp32 needs
//                    fp32 products, which the bf16 tensor-core path does not give.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "sm100.cuh"
#include "ws_header.cuh"

namespace flce {

constexpr int kStatusBadLabel = 5;  // FLCE_ERR_LABEL_OUT_OF_RANGE

__global__ void labels_kernel(const int64_t* __restrict__ labels, int64_t BT, int64_t V,
                              int64_t ignore_index, WsHeader* hdr) {
  __shared__ long long s_cnt[32];
  __shared__ int s_bad;
  if (threadIdx.x == 0) s_bad = 0;
  __syncthreads();
  long long cnt = 0;
  int bad = 0;
  for (int64_t i = threadIdx.x; i < BT; i += blockDim.x) {
    const int64_t l = labels[i];
    if (l != ignore_index) {
      ++cnt;
      if (l < 0 || l >= V) bad = 1;
    }
  }
  if (bad) s_bad = 1;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_down_sync(0xffffffffu, cnt, o);
  if ((threadIdx.x & 31) == 0) s_cnt[threadIdx.x >> 5] = cnt;
  __syncthreads();
  if (threadIdx.x == 0) {
    long long tot = 0;
    for (int w = 0; w < int(blockDim.x >> 5); ++w) tot += s_cnt[w];
    hdr->n_valid = tot;
    hdr->status = s_bad ? kStatusBadLabel : 0;
  }
}

// Label of row i when the op shifts token ids itself (T > 0): position t of
// each T-position sequence is scored against the id at t + 1; the last
// position has none and is ignored.
__device__ __forceinline__ int64_t shifted_label(const int64_t* __restrict__ ids, int64_t i,
                                                 int64_t T, int64_t ignore_index) {
  if (T <= 0) return ids[i];
  return (i % T == T - 1) ? ignore_index : ids[i + 1];
}

// The op's own copy of the shifted labels, which every later kernel reads.
__global__ void shift_labels_kernel(const int64_t* __restrict__ ids, int64_t BT, int64_t T,
                                    int64_t ignore_index, int64_t* __restrict__ out) {
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < BT;
       i += int64_t(gridDim.x) * blockDim.x)
    out[i] = shifted_label(ids, i, T, ignore_index);
}

// Data parallelism over rows: the number of rows whose label is not
// ignore_index (labels out of range are counted too; the loss call flags
// them), after the shift when T > 0, summed in a fixed order by one block.
__global__ void count_valid_kernel(const int64_t* __restrict__ labels, int64_t BT, int64_t T,
                                   int64_t ignore_index, int64_t* __restrict__ out) {
  __shared__ long long s_cnt[32];
  long long cnt = 0;
  for (int64_t i = threadIdx.x; i < BT; i += blockDim.x)
    cnt += shifted_label(labels, i, T, ignore_index) != ignore_index;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_down_sync(0xffffffffu, cnt, o);
  if ((threadIdx.x & 31) == 0) s_cnt[threadIdx.x >> 5] = cnt;
  __syncthreads();
  if (threadIdx.x == 0) {
    long long tot = 0;
    for (int w = 0; w < int(blockDim.x >> 5); ++w) tot += s_cnt[w];
    *out = tot;
  }
}

// The mean's divisor from outside the call (the count over all data-parallel
// ranks): replaces the call's own count once the labels check has run.
__global__ void set_n_valid_kernel(WsHeader* hdr, const int64_t* __restrict__ n_valid) {
  if (hdr->status == 0) hdr->n_valid = *n_valid;
}

// One thread per row.  partial is [n_tiles][BT] of (max of y*log2e, sum exp2(.-max)).
__global__ void combine_kernel(const float2* __restrict__ partial, int n_tiles, int64_t BT,
                               const float* __restrict__ target,
                               const int64_t* __restrict__ labels, int64_t ignore_index,
                               float* __restrict__ lse, float* __restrict__ row_loss,
                               const WsHeader* hdr) {
  const int64_t row = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (row >= BT || hdr->status != 0) return;
  float m = -INFINITY;
  for (int t = 0; t < n_tiles; ++t) m = fmaxf(m, partial[size_t(t) * BT + row].x);
  float s = 0.f;
  for (int t = 0; t < n_tiles; ++t) {
    const float2 p = partial[size_t(t) * BT + row];
    s += p.y * exp2f(p.x - m);
  }
  const float l = (m + log2f(s)) * 0.69314718055994531f;
  lse[row] = l;
  row_loss[row] = (labels[row] != ignore_index) ? l - target[row] : 0.f;
}

// Vocabulary parallelism, one rank's slice [v_off, v_off + n_cols) of the
// vocabulary: per row, fold the forward GEMM's per-tile partials into the
// slice's (largest y log2 e, sum of exp2(y log2 e - that), y at the label
// when the label lies in the slice else 0), stats [BT][3].  Rows of another
// rank's label and ignored rows still get the slice's max and sum.
__global__ void vp_stats_kernel(const float2* __restrict__ partial, int n_tiles, int64_t BT,
                                const float* __restrict__ target,
                                const int64_t* __restrict__ labels, int64_t ignore_index,
                                int64_t v_off, int64_t n_cols, float* __restrict__ stats,
                                const WsHeader* hdr) {
  const int64_t row = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (row >= BT || hdr->status != 0) return;
  float m = -INFINITY;
  for (int t = 0; t < n_tiles; ++t) m = fmaxf(m, partial[size_t(t) * BT + row].x);
  float s = 0.f;
  for (int t = 0; t < n_tiles; ++t) {
    const float2 p = partial[size_t(t) * BT + row];
    s += p.y * exp2f(p.x - m);
  }
  const int64_t lab = labels[row];
  const bool here = lab != ignore_index && lab >= v_off && lab < v_off + n_cols;
  stats[row * 3] = m;
  stats[row * 3 + 1] = s;
  stats[row * 3 + 2] = here ? target[row] : 0.f;
}

// Vocabulary parallelism: the ranks' slice statistics [n_ranks][BT][3],
// combined per row in rank order: M = max of the maxima, S = sum of
// s_r exp2(m_r - M), the target from the rank that holds it; lse and the
// row's NLL (the mean follows in finalize_kernel).
__global__ void vp_combine_kernel(const float* __restrict__ stats, int n_ranks, int64_t BT,
                                  const int64_t* __restrict__ labels, int64_t ignore_index,
                                  float* __restrict__ lse, float* __restrict__ row_loss,
                                  const WsHeader* hdr) {
  const int64_t row = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (row >= BT || hdr->status != 0) return;
  const size_t rs = size_t(BT) * 3;
  float M = -INFINITY;
  for (int r = 0; r < n_ranks; ++r) M = fmaxf(M, stats[r * rs + row * 3]);
  float S = 0.f, tgt = 0.f;
  for (int r = 0; r < n_ranks; ++r) {
    const float* st = stats + r * rs + row * 3;
    S += st[1] * exp2f(st[0] - M);
    tgt += st[2];
  }
  const float l = (M + log2f(S)) * 0.69314718055994531f;
  lse[row] = l;
  row_loss[row] = labels[row] != ignore_index ? l - tgt : 0.f;
}

__global__ void finalize_kernel(const float* __restrict__ row_loss, int64_t BT,
                                const WsHeader* hdr, float* loss) {
  __shared__ double sh[1024];
  double acc = 0.0;
  for (int64_t i = threadIdx.x; i < BT; i += blockDim.x) acc += double(row_loss[i]);
  sh[threadIdx.x] = acc;
  __syncthreads();
  for (int w = blockDim.x / 2; w > 0; w >>= 1) {
    if (int(threadIdx.x) < w) sh[threadIdx.x] += sh[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const long long nv = hdr->n_valid;
    *loss = (hdr->status == 0 && nv > 0) ? float(sh[0] / double(nv)) : (nv > 0 ? NAN : 0.f);
  }
}

// Fused-in-forward schedule, after a row chunk's forward GEMM.  Every row's
// partials -- per vocabulary slice the largest u = y log2(e) and the sum of
// exp2(u - R) -- share the row's one reference R (0, or the row's maximum
// after a recomputation), so for each row of the chunk:
//   S = sum over slices of the sums (in slice order), lse = (R + log2 S) ln 2,
//   the row's NLL, f = exp2(R - log2 S - R) = 1 / S (0 for an ignored row),
//   row_scale = f dloss / N (the dX epilogue's factor),
//   Xs = bf16(f x) (the dW GEMM's operand), and the label column of the
//   chunk buffer replaced by (p - 1) dy/dz / f -- G / (f dloss / N) there,
//   computed from the fp32 target logit so a probability near 1 loses
//   nothing -- after which G = (dloss / N) diag(f) Q everywhere.
// q, f and Xs stay inside bf16's normal range while the row's largest u lies
// in [-kRefWindow, kRefWindow]; a valid row outside it (or with a sum that is
// not finite) is left by pass 1, which records its exact maximum as its new
// reference and flags its 32-row group (every other row keeps reference 0).
// The forward GEMM then recomputes the flagged groups against those
// references -- rewriting their rows of P whole, label columns included --
// and pass 2 finishes every row of the flagged groups (blocks of unflagged
// groups return at once); a row that was fine gets the same values again.
constexpr int kLseQRows = 32;       // rows per block: one flag group
constexpr int kLseQThreads = 512;   // sixteen warps; lane = row of the group
constexpr float kRefWindow = 64.f;  // log2 units

__global__ void __launch_bounds__(kLseQThreads)
    lse_q_kernel(int pass, const float2* __restrict__ partial, int n_parts, int64_t BT,
                 int64_t row0, int64_t rows, const float* __restrict__ target,
                 const int64_t* __restrict__ labels, int64_t ignore_index,
                 __nv_bfloat16* __restrict__ P, int64_t ldp, const __nv_bfloat16* __restrict__ X,
                 int64_t ldx, int64_t H, __nv_bfloat16* __restrict__ Xs, float* __restrict__ ref,
                 int* __restrict__ group_flags,
                 float* __restrict__ lse_out, float* __restrict__ row_loss,
                 float* __restrict__ row_scale, const WsHeader* hdr, float dloss,
                 float softcap) {
  __shared__ float s_max[kLseQThreads / 32][kLseQRows];
  __shared__ float s_sum[kLseQThreads / 32][kLseQRows];
  __shared__ float s_f[kLseQRows];
  __shared__ int s_do[kLseQRows];  // this pass finishes the row
  if (hdr->status != 0) return;
  const int group = blockIdx.x;
  if (pass == 2 && group_flags[group] == 0) return;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const int64_t lrow = int64_t(group) * kLseQRows + lane;
  const bool in = lrow < rows;
  const int64_t row = row0 + lrow;
  // ---- per row: max and sum of the partials; warp w takes slices w, w+16,
  // ..., eight loads in flight
  constexpr int kW = kLseQThreads / 32;
  float m = -INFINITY, sum = 0.f;
  if (in) {
    const float2* pr = partial + row;
    for (int t = wid; t < n_parts; t += 8 * kW) {
      float2 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int tt = t + u * kW;
        v[u] = tt < n_parts ? pr[size_t(tt) * BT] : make_float2(-INFINITY, 0.f);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        m = fmaxf(m, v[u].x);
        sum += v[u].y;
      }
    }
  }
  s_max[wid][lane] = m;
  s_sum[wid][lane] = sum;
  __syncthreads();
  if (wid == 0) {
    float M = s_max[0][lane], S = s_sum[0][lane];
    for (int w = 1; w < kW; ++w) {
      M = fmaxf(M, s_max[w][lane]);
      S += s_sum[w][lane];
    }
    const int64_t lab = in ? labels[row] : ignore_index;
    const bool keep = lab != ignore_index;
    bool finish = in;
    float f = 0.f;
    if (finish) {
      const float R = pass == 1 ? 0.f : ref[lrow];
      const bool ok = M >= -kRefWindow && M <= kRefWindow && S < INFINITY;
      if (pass == 1 && keep && !ok) {
        ref[lrow] = M;  // recompute against the row's exact maximum
        finish = false;
      } else {
        if (pass == 1) ref[lrow] = 0.f;
        const float lse2 = R + log2f(S);
        const float l = lse2 * 0.69314718055994531f;
        lse_out[row] = l;
        const float tgt = keep ? target[row] : 0.f;
        row_loss[row] = keep ? l - tgt : 0.f;
        const long long nv = hdr->n_valid;
        f = keep ? 1.f / S : 0.f;
        row_scale[lrow] = keep && nv > 0 ? f * (dloss / float(nv)) : 0.f;
        if (keep) {
          float d = 1.f;
          if (softcap > 0.f) {
            const float t = tgt / softcap;
            d = 1.f - t * t;
          }
          const float p = exp2f(fmaf(tgt, 1.4426950408889634f, -lse2));
          P[lrow * ldp + lab] = __float2bfloat16_rn((p - 1.f) * d * S);
        }
      }
    }
    s_do[lane] = finish ? 1 : 0;
    s_f[lane] = f;
    const unsigned any = __ballot_sync(0xffffffffu, pass == 1 && in && keep && !finish);
    if (pass == 1 && lane == 0) group_flags[group] = any != 0u;
  }
  __syncthreads();
  // ---- Xs = bf16(f x) for the rows this pass finished: 8 columns per
  // thread and step, two steps' loads in flight
  const int64_t vecs = H / 8;
  const int64_t items = int64_t(kLseQRows) * vecs;
  for (int64_t e0 = tid; e0 < items; e0 += 2 * kLseQThreads) {
    uint4 raw[2];
    int rr[2];
    int64_t k[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int64_t e = e0 + int64_t(u) * kLseQThreads;
      rr[u] = e < items ? int(e / vecs) : 0;
      k[u] = (e - int64_t(rr[u]) * vecs) * 8;
      if (e < items && s_do[rr[u]])
        raw[u] = *reinterpret_cast<const uint4*>(
            X + (row0 + int64_t(group) * kLseQRows + rr[u]) * ldx + k[u]);
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int64_t e = e0 + int64_t(u) * kLseQThreads;
      if (e >= items || !s_do[rr[u]]) continue;
      const float f = s_f[rr[u]];
      __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&raw[u]);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 v = __bfloat1622float2(h[q]);
        h[q] = __floats2bfloat162_rn(v.x * f, v.y * f);
      }
      *reinterpret_cast<uint4*>(Xs + (int64_t(group) * kLseQRows + rr[u]) * H + k[u]) = raw[u];
    }
  }
}

// dX rows of a row chunk from its K-split slabs: out = bf16(sum_s slab_s *
// row_scale[row]), summed in split order (row_scale null: 1).  The slabs are
// dense rows of H; output rows are ld_out apart.  n (rows * H) and H are
// multiples of 8, as is ld_out.
__global__ void slab_reduce_kernel(const float* __restrict__ slabs, int n_slabs,
                                   int64_t slab_stride, int64_t n, int64_t H,
                                   __nv_bfloat16* __restrict__ out, int64_t ld_out,
                                   const float* __restrict__ row_scale, const WsHeader* hdr) {
  if (hdr->status != 0) return;
  for (int64_t i = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) * 8; i < n;
       i += int64_t(gridDim.x) * blockDim.x * 8) {
    float4 a = *reinterpret_cast<const float4*>(slabs + i);
    float4 b = *reinterpret_cast<const float4*>(slabs + i + 4);
    for (int sidx = 1; sidx < n_slabs; ++sidx) {
      const float* p = slabs + int64_t(sidx) * slab_stride + i;
      const float4 c = *reinterpret_cast<const float4*>(p);
      const float4 d = *reinterpret_cast<const float4*>(p + 4);
      a.x += c.x; a.y += c.y; a.z += c.z; a.w += c.w;
      b.x += d.x; b.y += d.y; b.z += d.z; b.w += d.w;
    }
    const float f = row_scale ? row_scale[i / H] : 1.f;
    __nv_bfloat162 h[4] = {__floats2bfloat162_rn(a.x * f, a.y * f),
                           __floats2bfloat162_rn(a.z * f, a.w * f),
                           __floats2bfloat162_rn(b.x * f, b.y * f),
                           __floats2bfloat162_rn(b.z * f, b.w * f)};
    *reinterpret_cast<uint4*>(out + (i / H) * ld_out + i % H) = *reinterpret_cast<uint4*>(h);
  }
}

// Failure-path self-test: wait, with the library's bounded wait, on an
// mbarrier that nothing will ever arrive on; the wait gives up after
// limit_ns and the kernel records the timeout in the status word.
constexpr int kStatusTimeoutAux = 6;  // FLCE_ERR_TIMEOUT

__global__ void selftest_wait_kernel(WsHeader* hdr, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  fence_barrier_init();
  if (!mbar_wait_bounded(&bar, 0, limit_ns, nullptr)) atomicCAS(&hdr->status, 0, kStatusTimeoutAux);
}

// ------------------------------ SIMT path ----------------------------------
// 32x32 output tiles, 32x8 threads, each thread four rows of one column.

template <typename T>
__device__ __forceinline__ float ld_f(const T* p);
template <>
__device__ __forceinline__ float ld_f<float>(const float* p) { return *p; }
template <>
__device__ __forceinline__ float ld_f<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}
template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

struct SimtEpi {
  const WsHeader* hdr;
  const int64_t* labels;
  int64_t ignore_index;
  int64_t BT, H, V;
  int64_t ldx, ldw, lddx, lddw;  // row strides of X, W, dX, dW (elements)
  int64_t label_off;             // vocabulary id of W's first row (labels are global)
  float softcap;
  // logits modes
  float2* partial;         // [ceil(V/32)][BT]
  float* target;
  const float* lse;
  const float* dloss_dev;
  float dloss_host;
  float* G;                // fp32 chunk buffer, row stride ldg
  int64_t ldg;
  int64_t v0;              // chunk's first vocabulary index
  int64_t chunk;           // chunk width (columns of G actually used)
  // gemm modes
  float* dx_acc;
  void* dx;
  int dx_first, dx_last;
  void* dw;
};

// Logit tiles Z = X W^T for vocabulary columns [v0 + 32*bx, +32).
// MODE 0: online-LSE partials; MODE 1: G into the chunk buffer.
template <typename T, int MODE>
__global__ void simt_logits_kernel(const T* __restrict__ X, const T* __restrict__ W,
                                   SimtEpi ep) {
  __shared__ float xs[32][33];
  __shared__ float ws[32][33];
  if (ep.hdr->status != 0) return;
  const int tx = threadIdx.x, ty = threadIdx.y;
  const int64_t m0 = int64_t(blockIdx.y) * 32;
  const int64_t n0 = int64_t(blockIdx.x) * 32;  // relative to v0
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int64_t k0 = 0; k0 < ep.H; k0 += 32) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int rr = ty + 8 * i;
      const int64_t xr = m0 + rr, wr = ep.v0 + n0 + rr, kk = k0 + tx;
      xs[rr][tx] = (xr < ep.BT && kk < ep.H) ? ld_f(X + xr * ep.ldx + kk) : 0.f;
      ws[rr][tx] = (wr < ep.V && kk < ep.H) ? ld_f(W + wr * ep.ldw + kk) : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < 32; ++kk) {
      const float w = ws[tx][kk];
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[i] = fmaf(xs[ty + 8 * i][kk], w, acc[i]);
    }
    __syncthreads();
  }
  const bool cap = ep.softcap > 0.f;
  const int64_t j = ep.v0 + n0 + tx;  // vocabulary column of this thread
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t row = m0 + ty + 8 * i;
    if (row >= ep.BT) continue;  // uniform across the warp (one row per warp)
    const float z = acc[i];
    const float t = cap ? tanhf(z / ep.softcap) : 0.f;
    const float y = cap ? ep.softcap * t : z;
    const int64_t lab = ep.labels[row];
    if (MODE == 0) {
      const float u = (j < ep.V) ? y * 1.4426950408889634f : -INFINITY;
      float m = u;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      float s = exp2f(u - m);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (tx == 0) ep.partial[size_t(blockIdx.x) * ep.BT + row] = make_float2(m, s);
      if (lab == j + ep.label_off && lab != ep.ignore_index) ep.target[row] = y;
    } else {
      const long long nv = ep.hdr->n_valid;
      const bool valid = lab != ep.ignore_index && nv > 0;
      float g = 0.f;
      if (valid && j < ep.V) {
        const float dl = ep.dloss_dev ? *ep.dloss_dev : ep.dloss_host;
        const float p = expf(y - ep.lse[row]);
        const float d = cap ? 1.f - t * t : 1.f;
        g = (p - (j + ep.label_off == lab ? 1.f : 0.f)) * d * (dl / float(nv));
      }
      if (n0 + tx < ep.ldg) ep.G[row * ep.ldg + n0 + tx] = g;
    }
  }
}

// MODE 2 (dX):  C[BT x H] = G[BT x chunk] * W[v0 .. v0+chunk, :]
// MODE 3 (dW):  C[chunk x H] = G^T * X, rows v0.. of dW
template <typename T, int MODE>
__global__ void simt_gemm_kernel(const T* __restrict__ Bsrc, SimtEpi ep) {
  __shared__ float as[32][33];  // [m][k]
  __shared__ float bs[32][33];  // [k][n]
  if (ep.hdr->status != 0) return;
  const int tx = threadIdx.x, ty = threadIdx.y;
  const int64_t m0 = int64_t(blockIdx.y) * 32;
  const int64_t n0 = int64_t(blockIdx.x) * 32;
  const int64_t Mrows = (MODE == 2) ? ep.BT : ep.chunk;
  const int64_t Kdim = (MODE == 2) ? ep.chunk : ep.BT;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int64_t k0 = 0; k0 < Kdim; k0 += 32) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int rr = ty + 8 * i;
      if (MODE == 2) {
        const int64_t gr = m0 + rr, gc = k0 + tx;  // G[row][col]
        as[rr][tx] = (gr < ep.BT && gc < ep.chunk) ? ep.G[gr * ep.ldg + gc] : 0.f;
        const int64_t wr = k0 + rr, wc = n0 + tx;  // W[v0 + wr][wc]
        bs[rr][tx] = (wr < ep.chunk && ep.v0 + wr < ep.V && wc < ep.H)
                         ? ld_f(Bsrc + (ep.v0 + wr) * ep.ldw + wc) : 0.f;
      } else {
        const int64_t gk = k0 + rr, gm = m0 + tx;  // G[gk][gm] is A[gm][gk]
        as[tx][rr] = (gk < ep.BT && gm < ep.chunk) ? ep.G[gk * ep.ldg + gm] : 0.f;
        const int64_t xr = k0 + rr, xc = n0 + tx;
        bs[rr][tx] = (xr < ep.BT && xc < ep.H) ? ld_f(Bsrc + xr * ep.ldx + xc) : 0.f;
      }
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < 32; ++kk) {
      const float b = bs[kk][tx];
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[i] = fmaf(as[ty + 8 * i][kk], b, acc[i]);
    }
    __syncthreads();
  }
  const int64_t col = n0 + tx;
  if (col >= ep.H) return;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t row = m0 + ty + 8 * i;
    if (row >= Mrows) continue;
    if (MODE == 2) {
      float a = acc[i];
      float* p = ep.dx_acc + row * ep.H + col;
      if (!ep.dx_first) a += *p;
      if (!ep.dx_last)
        *p = a;
      else
        static_cast<T*>(ep.dx)[row * ep.lddx + col] = from_f<T>(a);
    } else {
      const int64_t v = ep.v0 + row;
      if (v < ep.V) static_cast<T*>(ep.dw)[v * ep.lddw + col] = from_f<T>(acc[i]);
    }
  }
}

}  // namespace flce

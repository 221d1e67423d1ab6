// ce_kernels.cuh -- cross-entropy for a caller that already holds the logits.
//
// PyTorch PR #126348 ("[AOTAutograd] tweak min-cut partitioner to avoid
// saving softmax output") lists the unfused loss as four passes over the
// BT x V softmax_input: the matmul, a row max, a row sum, and a normalised
// softmax_output saved for backward.  Its points a. and b.: the forward
// needs only the label's entry of the softmax, and the backward can rebuild
// the softmax from softmax_input and the small row statistics instead of
// reading a saved one.  These kernels are that plan on a B200:
//
//   ce_forward_kernel   one read of each logits row: online max / sum-exp in
//                       registers, a fixed-order block combine, lse and the
//                       row's NLL.  No softmax is written.
//   ce_backward_kernel  one read of each logits row and one write of its
//                       gradient G = (exp(y - lse) - onehot) * dy/dz *
//                       dloss / N, the softmax rebuilt from the logits and
//                       the saved lse; may run in place (dlogits == logits).
//
// Both are HBM-bound: the bytes are the logits (and the gradient), the
// arithmetic one exp2 per element (two more with a softcap).  One block of
// kCeThreads threads per row streams 16-byte vectors, kCeUnroll loads in
// flight per thread.  A row that does not start on a 16-byte boundary (an odd
// V in a dense bf16 tensor) takes its first elements up to the boundary, and
// its last elements past the final whole vector, one element per thread.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "gemm_tc.cuh"
#include "ws_header.cuh"

namespace flce {

constexpr int kCeThreads = 256;
constexpr int kCeUnroll = 4;

template <typename T>
struct CeElem;
template <>
struct CeElem<__nv_bfloat16> {
  static constexpr int kVec = 8;  // elements per 16-byte vector
  __device__ static float get(const uint4& v, int k) {
    const uint32_t w = (&v.x)[k >> 1];
    return __uint_as_float((k & 1) ? (w & 0xffff0000u) : (w << 16));
  }
  __device__ static float one(const __nv_bfloat16* p) { return __bfloat162float(*p); }
  __device__ static void put(uint4& v, int k, float lo, float hi) {  // k even
    (&v.x)[k >> 1] = pack_bf16x2(lo, hi);
  }
  __device__ static void store_one(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }
  // Largest of the 8 values, compared as packed bf16 pairs.
  __device__ static float vmax(const uint4& v) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
    const __nv_bfloat162 a = __hmax2(__hmax2(h[0], h[1]), __hmax2(h[2], h[3]));
    return fmaxf(__low2float(a), __high2float(a));
  }
  __device__ static uint4 neg_inf() {  // 8 x bf16 -inf
    return make_uint4(0xff80ff80u, 0xff80ff80u, 0xff80ff80u, 0xff80ff80u);
  }
};
template <>
struct CeElem<float> {
  static constexpr int kVec = 4;
  __device__ static float get(const uint4& v, int k) { return __uint_as_float((&v.x)[k]); }
  __device__ static float one(const float* p) { return *p; }
  __device__ static void put(uint4& v, int k, float lo, float hi) {
    (&v.x)[k] = __float_as_uint(lo);
    (&v.x)[k + 1] = __float_as_uint(hi);
  }
  __device__ static void store_one(float* p, float x) { *p = x; }
  __device__ static float vmax(const uint4& v) {
    return fmaxf(fmaxf(__uint_as_float(v.x), __uint_as_float(v.y)),
                 fmaxf(__uint_as_float(v.z), __uint_as_float(v.w)));
  }
  __device__ static uint4 neg_inf() {
    const uint32_t n = 0xff800000u;
    return make_uint4(n, n, n, n);
  }
};

// Elements of a row before its first 16-byte boundary (at most V).
template <typename T>
__device__ __forceinline__ int64_t ce_head(const T* row, int64_t V) {
  const int64_t h = int64_t((16u - (reinterpret_cast<uintptr_t>(row) & 15u)) & 15u) / sizeof(T);
  return h < V ? h : V;
}

// y * log2(e), with y = c tanh(z / c) under a softcap.
template <bool CAP>
__device__ __forceinline__ float ce_u(float z, float sc, float inv_sc) {
  float d;
  return capped<CAP>(z, sc, inv_sc, &d) * kLog2e;
}

// Online (max, sum of exp2(u - max)) of one thread: fold in a group whose
// largest u is gmax; `add` sums the group's exp2(u - m) for the new m.
__device__ __forceinline__ void ce_merge(float& m, float& s, float m2, float s2) {
  const float mn = fmaxf(m, m2);
  if (mn == -INFINITY) return;  // nothing but empty or -inf entries so far
  s = s * ex2a(m - mn) + s2 * ex2a(m2 - mn);
  m = mn;
}

// Combine the 32 lanes' (max, sum of exp2(u - max)) pairs: the max by an
// xor butterfly, each lane's sum rescaled to it (one exp2), the sums by a
// second butterfly.  Every step is symmetric in its two operands, so all
// lanes end with the same bits.  An empty lane is (-inf, 0).
__device__ __forceinline__ void ce_warp_combine(float& m, float& s) {
  float M = m;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  float S = (m == -INFINITY) ? 0.f : s * ex2a(m - M);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) S += __shfl_xor_sync(0xffffffffu, S, o);
  m = M;
  s = S;
}

template <typename T, bool CAP>
__global__ void __launch_bounds__(kCeThreads)
    ce_forward_kernel(const T* __restrict__ Z, int64_t ld, int64_t V,
                      const int64_t* __restrict__ labels, int64_t ignore_index, float softcap,
                      float* __restrict__ lse_out, float* __restrict__ row_loss,
                      const WsHeader* hdr) {
  using E = CeElem<T>;
  constexpr int VE = E::kVec;
  __shared__ float red_m[kCeThreads / 32], red_s[kCeThreads / 32];
  if (hdr->status != 0) return;
  const int64_t row = blockIdx.x;
  const int tid = threadIdx.x;
  const T* z = Z + row * ld;
  const float sc = softcap;
  const float inv_sc = CAP ? 1.f / softcap : 0.f;
  const int64_t head = ce_head(z, V);
  const int64_t nvec = (V - head) / VE;
  const int64_t tail0 = head + nvec * VE;
  float m = -INFINITY, s = 0.f;
  // Scalar elements: the head and the tail, one per thread.
  for (int64_t j = tid; j < head + (V - tail0); j += kCeThreads) {
    const int64_t col = j < head ? j : tail0 + (j - head);
    const float u = ce_u<CAP>(E::one(z + col), sc, inv_sc);
    ce_merge(m, s, u, 1.f);
  }
  const uint4* zv = reinterpret_cast<const uint4*>(z + head);
  for (int64_t v0 = tid; v0 < nvec; v0 += int64_t(kCeUnroll) * kCeThreads) {
    uint4 raw[kCeUnroll];
#pragma unroll
    for (int u = 0; u < kCeUnroll; ++u) {
      const int64_t v = v0 + int64_t(u) * kCeThreads;
      if (v < nvec) raw[u] = __ldcs(zv + v);
    }
    // The group's largest logit (the softcap is increasing, so it caps the
    // largest raw value); bf16 pairs compare packed.  Vectors past the row
    // were not loaded: -inf.
    float gz = -INFINITY;
#pragma unroll
    for (int u = 0; u < kCeUnroll; ++u) {
      if (v0 + int64_t(u) * kCeThreads >= nvec) raw[u] = E::neg_inf();
      gz = fmaxf(gz, E::vmax(raw[u]));
    }
    if (gz == -INFINITY) continue;
    const float mn = fmaxf(m, ce_u<CAP>(gz, sc, inv_sc));
    float a0 = 0.f, a1 = 0.f;
#pragma unroll
    for (int u = 0; u < kCeUnroll; ++u) {
      if (v0 + int64_t(u) * kCeThreads >= nvec) break;  // not loaded (a capped -inf is not 0)
#pragma unroll
      for (int k = 0; k < VE; k += 2) {
        float d;
        a0 += ex2a(fmaf(capped<CAP>(E::get(raw[u], k), sc, inv_sc, &d), kLog2e, -mn));
        a1 += ex2a(fmaf(capped<CAP>(E::get(raw[u], k + 1), sc, inv_sc, &d), kLog2e, -mn));
      }
    }
    s = s * ex2a(m - mn) + (a0 + a1);
    m = mn;
  }
  // Fixed-order combine: warp butterflies, then warp 0 over the warps.
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
    const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
    ce_merge(m, s, m2, s2);
  }
  if ((tid & 31) == 0) {
    red_m[tid >> 5] = m;
    red_s[tid >> 5] = s;
  }
  __syncthreads();
  if (tid == 0) {
    float M = red_m[0], S = red_s[0];
    for (int w = 1; w < kCeThreads / 32; ++w) ce_merge(M, S, red_m[w], red_s[w]);
    const float l = (M + log2f(S)) * kLn2;
    const int64_t lab = labels[row];
    const bool valid = lab != ignore_index;
    float yt = 0.f;
    if (valid) {
      float d;
      yt = capped<CAP>(E::one(z + lab), sc, inv_sc, &d);
    }
    lse_out[row] = l;
    row_loss[row] = valid ? l - yt : 0.f;
  }
}

// G for one element: (exp(y - lse) - [label]) * dy/dz * scale, evaluated as
// p * s - [label] * s with s = dy/dz * scale -- the same operations as the
// vector form below, so an element gets the same bits on either path.
template <bool CAP>
__device__ __forceinline__ float ce_grad(float z, float sc, float inv_sc, float lse2, float scale,
                                         bool is_label) {
  float d;
  const float y = capped<CAP>(z, sc, inv_sc, &d);
  const float sd = CAP ? d * scale : scale;
  const float g = ex2a(fmaf(y, kLog2e, -lse2)) * sd;
  return is_label ? g - sd : g;
}

// G for the VE elements of one 16-byte vector, the one-hot term left out:
// exp(y - lse) * dy/dz * scale.  ce_vec_label then subtracts dy/dz * scale
// at the label, when the label falls in this vector (rel in [0, VE)): one
// comparison per vector instead of one per element.
template <typename T, bool CAP>
__device__ __forceinline__ void ce_vec_grad(const uint4& raw, float sc, float inv_sc, float lse2,
                                            float scale, float (&gg)[CeElem<T>::kVec]) {
#pragma unroll
  for (int k = 0; k < CeElem<T>::kVec; ++k) {
    float d;
    const float y = capped<CAP>(CeElem<T>::get(raw, k), sc, inv_sc, &d);
    gg[k] = ex2a(fmaf(y, kLog2e, -lse2)) * (CAP ? d * scale : scale);
  }
}
template <typename T, bool CAP>
__device__ __forceinline__ void ce_vec_label(const uint4& raw, int rel, float sc, float inv_sc,
                                             float scale, float (&gg)[CeElem<T>::kVec]) {
  if (unsigned(rel) >= unsigned(CeElem<T>::kVec)) return;
#pragma unroll
  for (int k = 0; k < CeElem<T>::kVec; ++k)
    if (k == rel) {
      float d;
      capped<CAP>(CeElem<T>::get(raw, k), sc, inv_sc, &d);
      gg[k] -= CAP ? d * scale : scale;
    }
}
// The label's position relative to the first vector of a row, as a 32-bit
// offset (V < 2^31); a label before the vectors (in the row's head) or an
// ignored row gives a value no vector matches.
__device__ __forceinline__ int ce_lab_rel(int64_t lab, int64_t head, bool valid) {
  return (valid && lab >= head) ? int(lab - head) : -1;
}

template <typename T, bool CAP>
__global__ void __launch_bounds__(kCeThreads)
    ce_backward_kernel(const T* Z, int64_t ld, T* dZ, int64_t ld_g, int64_t V,
                       const int64_t* __restrict__ labels, int64_t ignore_index, float softcap,
                       const float* __restrict__ lse, const float* __restrict__ dloss,
                       const WsHeader* hdr) {
  using E = CeElem<T>;
  constexpr int VE = E::kVec;
  if (hdr->status != 0) return;
  const int64_t row = blockIdx.x;
  const int tid = threadIdx.x;
  const T* z = Z + row * ld;
  T* g = dZ + row * ld_g;
  const int64_t lab = labels[row];
  const long long nv = hdr->n_valid;
  const bool valid = lab != ignore_index;
  const float scale = (valid && nv > 0) ? *dloss / float(nv) : 0.f;
  const float lse2 = scale != 0.f ? lse[row] * kLog2e : 0.f;
  const float sc = softcap;
  const float inv_sc = CAP ? 1.f / softcap : 0.f;
  // Vector loads and stores need the input and output rows to share their
  // 16-byte phase (in place, or both dense with the same row stride);
  // otherwise every element goes singly.
  const int64_t head = ce_head(z, V);
  const bool same_phase = ce_head(g, V) == head;
  const int64_t nvec = same_phase ? (V - head) / VE : 0;
  const int64_t lo = same_phase ? head : V;   // scalar elements: [0, lo) and [hi, V)
  const int64_t hi = same_phase ? head + nvec * VE : V;
  for (int64_t j = tid; j < lo + (V - hi); j += kCeThreads) {
    const int64_t col = j < lo ? j : hi + (j - lo);
    const float x = scale != 0.f ? ce_grad<CAP>(E::one(z + col), sc, inv_sc, lse2, scale,
                                                 col == lab)
                                 : 0.f;
    E::store_one(g + col, x);
  }
  const uint4* zv = reinterpret_cast<const uint4*>(z + head);
  uint4* gv = reinterpret_cast<uint4*>(g + head);
  if (scale == 0.f) {  // ignored row, or no valid row at all: zeros
    for (int64_t v = tid; v < nvec; v += kCeThreads) __stcs(gv + v, make_uint4(0u, 0u, 0u, 0u));
    return;
  }
  const int lab_rel = ce_lab_rel(lab, head, valid);  // label's position in the vector run
  const int nv32 = int(nvec);
  for (int v0 = tid; v0 < nv32; v0 += kCeUnroll * kCeThreads) {
    uint4 raw[kCeUnroll];
#pragma unroll
    for (int u = 0; u < kCeUnroll; ++u) {
      const int v = v0 + u * kCeThreads;
      if (v < nv32) raw[u] = __ldcs(zv + v);
    }
#pragma unroll
    for (int u = 0; u < kCeUnroll; ++u) {
      const int v = v0 + u * kCeThreads;
      if (v >= nv32) break;
      float gg[VE];
      ce_vec_grad<T, CAP>(raw[u], sc, inv_sc, lse2, scale, gg);
      ce_vec_label<T, CAP>(raw[u], lab_rel - v * VE, sc, inv_sc, scale, gg);
      uint4 out;
#pragma unroll
      for (int k = 0; k < VE; k += 2) E::put(out, k, gg[k], gg[k + 1]);
      __stcs(gv + v, out);
    }
  }
}

}  // namespace flce

namespace flce {

// Forward and backward in one pass over HBM, for a caller that holds the
// logits and wants the loss and the logit gradient together: one read and
// one write of each row instead of two reads and a write.
//
// ce_fused_pipe_kernel (rows up to kCeFusedRowMax bytes): one persistent
// block per SM, two row buffers in shared memory, a producer warp and
// kCePipeWarps compute warps.
//   producer  brings the 16-byte aligned interior of each of the block's rows
//             into a buffer with one bulk asynchronous copy (completion
//             counted on the buffer's `full` mbarrier) as soon as every
//             compute warp has released the buffer (its `empty` mbarrier).
//   compute   per row: (max, sum-exp) of the row from shared memory; one named
//             barrier that also ANDs the warps' wait results; each warp merges
//             the warp partials itself in the same fixed tree (no second
//             barrier); the row's gradient written to global memory; the
//             buffer released, and on to the next row, whose copy has
//             usually landed by then.
// The few elements before the first and after the last 16-byte boundary of a
// row, and the label's logit, come from global memory through plain loads
// issued before the wait, so every access stays inside the row.  Waits are
// bounded: one that gives up records FLCE_ERR_TIMEOUT, the compute warps
// leave together, and the producer waits (bounded) for its copies still in
// flight before the block exits.
//
// ce_fused_rows_kernel (longer rows): one block per row, the row read twice
// (the second time mostly from L2, it was loaded moments before).  N_valid
// must be known (labels_kernel ran first); dloss is a host value.  dZ may be
// Z (in place).
#ifndef FLCE_CE_PIPE_WARPS
#define FLCE_CE_PIPE_WARPS 16
#endif
constexpr int kCePipeWarps = FLCE_CE_PIPE_WARPS;
static_assert(kCePipeWarps >= 1 && kCePipeWarps <= 31, "compute warps of one block, plus one");
constexpr int kCePipeThreads = (kCePipeWarps + 1) * 32;
constexpr int kCeFusedThreads = 512;
constexpr int kCeFusedRowMax = 112 * 1024;

template <typename T, bool CAP>
__global__ void __launch_bounds__(kCePipeThreads, 1)
    ce_fused_pipe_kernel(const T* Z, int64_t ld, T* dZ, int64_t ld_g, int64_t BT, int64_t V,
                         const int64_t* __restrict__ labels, int64_t ignore_index,
                         float softcap, float dloss, float* __restrict__ lse_out,
                         float* __restrict__ row_loss, WsHeader* hdr, uint32_t buf_bytes,
                         unsigned long long wait_limit_ns) {
  using E = CeElem<T>;
  constexpr int VE = E::kVec;
  constexpr int kW = kCePipeWarps;
  constexpr int kC = kW * 32;  // compute threads
  extern __shared__ __align__(128) uint8_t s_buf[];
  __shared__ uint64_t full[2], empty[2];
  __shared__ float red_m[2][kW], red_s[2][kW];
  __shared__ int s_skip;
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    // one reading of the status word for the whole block (another block may
    // set it while this one starts)
    s_skip = hdr->status != 0;
    mbar_init(&full[0], 1);
    mbar_init(&full[1], 1);
    mbar_init(&empty[0], kW);
    mbar_init(&empty[1], kW);
    fence_barrier_init();
  }
  __syncthreads();
  if (s_skip) return;
  const int64_t stride = gridDim.x;

  if (warp == kW) {
    // ---- producer (one thread)
    if (lane != 0) return;
    const uint64_t pol = policy_evict_first();
    bool ok = true;
    int64_t k = 0;  // copies issued
    for (int64_t row = blockIdx.x; row < BT; row += stride, ++k) {
      const int b = int(k & 1);
      // use k >> 1 of buffer b; the previous use must have been released
      if (k >= 2 &&
          !mbar_wait_bounded(&empty[b], uint32_t(((k >> 1) - 1) & 1), wait_limit_ns, nullptr)) {
        ok = false;
        break;
      }
      fence_proxy_async_smem();  // the released buffer's generic reads come first
      const T* z = Z + row * ld;
      const int64_t head = ce_head(z, V);
      const uint32_t bytes = uint32_t(((V - head) / VE) * 16);
      if (bytes) {
        mbar_arrive_expect_tx(&full[b], bytes);
        bulk_load_g2s(s_buf + size_t(b) * buf_bytes, z + head, bytes, &full[b], pol);
      } else {
        mbar_arrive(&full[b]);
      }
    }
    if (!ok) atomicCAS(&hdr->status, 0, kStatusTimeout);
    // the last copy into each buffer lands before the block's memory goes
    for (int64_t j = k >= 2 ? k - 2 : 0; j < k; ++j)
      mbar_wait_bounded(&full[j & 1], uint32_t((j >> 1) & 1), kDrainLimitNs, nullptr);
    return;
  }

  // ---- compute warps
  const float sc = softcap;
  const float inv_sc = CAP ? 1.f / softcap : 0.f;
  const long long nv = hdr->n_valid;
  int64_t k = 0;
  for (int64_t row = blockIdx.x; row < BT; row += stride, ++k) {
    const int b = int(k & 1);
    const T* z = Z + row * ld;
    T* g = dZ + row * ld_g;
    const int64_t head = ce_head(z, V);
    const int64_t nvec = (V - head) / VE;
    const int64_t tail0 = head + nvec * VE;
    const int64_t lab = labels[row];
    const bool valid = lab != ignore_index;
    // Plain loads, in flight during the wait: this thread's edge element (at
    // most 2 VE - 2 per row) and, for thread 0, the label's logit.
    int64_t edge_col = -1;
    float edge = 0.f;
    if (tid < head + (V - tail0)) {
      edge_col = tid < head ? tid : tail0 + (tid - head);
      edge = E::one(z + edge_col);
    }
    float zt = 0.f;
    if (tid == 0 && valid) zt = E::one(z + lab);
    const bool got = mbar_wait_bounded(&full[b], uint32_t((k >> 1) & 1), wait_limit_ns, nullptr);
    const uint4* sv = reinterpret_cast<const uint4*>(s_buf + size_t(b) * buf_bytes);
    // ---- the row's max and sum
    float m = -INFINITY, s = 0.f;
    if (edge_col >= 0) ce_merge(m, s, ce_u<CAP>(edge, sc, inv_sc), 1.f);
    const int nv_here = got ? int(nvec) : 0;  // a failed wait reads nothing
    for (int v0 = tid; v0 < nv_here; v0 += kCeUnroll * kC) {
      uint4 raw[kCeUnroll];
#pragma unroll
      for (int u = 0; u < kCeUnroll; ++u) {
        const int v = v0 + u * kC;
        raw[u] = v < nv_here ? sv[v] : E::neg_inf();
      }
      float gz = -INFINITY;
#pragma unroll
      for (int u = 0; u < kCeUnroll; ++u) gz = fmaxf(gz, E::vmax(raw[u]));
      if (gz == -INFINITY) continue;
      const float mn = fmaxf(m, ce_u<CAP>(gz, sc, inv_sc));
      float a0 = 0.f, a1 = 0.f;
#pragma unroll
      for (int u = 0; u < kCeUnroll; ++u) {
        if (v0 + u * kC >= nv_here) break;
#pragma unroll
        for (int kk = 0; kk < VE; kk += 2) {
          float d;
          a0 += ex2a(fmaf(capped<CAP>(E::get(raw[u], kk), sc, inv_sc, &d), kLog2e, -mn));
          a1 += ex2a(fmaf(capped<CAP>(E::get(raw[u], kk + 1), sc, inv_sc, &d), kLog2e, -mn));
        }
      }
      s = s * ex2a(m - mn) + (a0 + a1);
      m = mn;
    }
    // The warp's (max, sum): the largest max by one butterfly, every lane's
    // sum rescaled to it once, then summed by a second butterfly (each step
    // symmetric, so every lane holds the same bits).
    ce_warp_combine(m, s);
    if (lane == 0) {
      red_m[b][warp] = m;
      red_s[b][warp] = s;
    }
    if (!bar_and(1, kC, got)) {  // every compute thread sees the same result
      if (tid == 0) atomicCAS(&hdr->status, 0, kStatusTimeout);
      return;
    }
    // Each warp combines the kW partials the same way (lanes past kW hold
    // the identity), so every lane and every warp gets the same bits.
    float M = lane < kW ? red_m[b][lane] : -INFINITY;
    float S = lane < kW ? red_s[b][lane] : 0.f;
    ce_warp_combine(M, S);
    const float lse2 = M + log2f(S);
    if (tid == 0) {
      const float l = lse2 * kLn2;
      float yt = 0.f;
      if (valid) {
        float d;
        yt = capped<CAP>(zt, sc, inv_sc, &d);
      }
      if (lse_out) lse_out[row] = l;
      row_loss[row] = valid ? l - yt : 0.f;
    }
    // ---- the row's gradient, from the buffer
    const float scale = (valid && nv > 0) ? dloss / float(nv) : 0.f;
    const float l2 = scale != 0.f ? lse2 : 0.f;
    if (edge_col >= 0)
      E::store_one(g + edge_col, scale != 0.f ? ce_grad<CAP>(edge, sc, inv_sc, l2, scale,
                                                             edge_col == lab)
                                              : 0.f);
    const bool same_phase = ce_head(g, V) == head;
    uint4* gv = reinterpret_cast<uint4*>(g + head);
    const int lab_rel = ce_lab_rel(lab, head, valid);
    const int nv32 = int(nvec);
    if (scale == 0.f) {  // ignored row, or no valid row at all: zeros
      for (int v = tid; v < nv32; v += kC) {
        if (same_phase) {
          __stcs(gv + v, make_uint4(0u, 0u, 0u, 0u));
        } else {
#pragma unroll
          for (int kk = 0; kk < VE; ++kk) E::store_one(g + head + int64_t(v) * VE + kk, 0.f);
        }
      }
    } else {
#pragma unroll 2
      for (int v = tid; v < nv32; v += kC) {
        const uint4 raw = sv[v];
        float gg[VE];
        ce_vec_grad<T, CAP>(raw, sc, inv_sc, l2, scale, gg);
        ce_vec_label<T, CAP>(raw, lab_rel - v * VE, sc, inv_sc, scale, gg);
        if (same_phase) {
          uint4 out;
#pragma unroll
          for (int kk = 0; kk < VE; kk += 2) E::put(out, kk, gg[kk], gg[kk + 1]);
          __stcs(gv + v, out);
        } else {
#pragma unroll
          for (int kk = 0; kk < VE; ++kk) E::store_one(g + head + int64_t(v) * VE + kk, gg[kk]);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[b]);  // this warp is done with the buffer
  }
}

template <typename T, bool CAP>
__global__ void __launch_bounds__(kCeFusedThreads)
    ce_fused_rows_kernel(const T* Z, int64_t ld, T* dZ, int64_t ld_g, int64_t V,
                    const int64_t* __restrict__ labels, int64_t ignore_index, float softcap,
                    float dloss, float* __restrict__ lse_out, float* __restrict__ row_loss,
                    const WsHeader* hdr) {
  using E = CeElem<T>;
  constexpr int VE = E::kVec;
  constexpr int kW = kCeFusedThreads / 32;
  __shared__ float red_m[kW], red_s[kW];
  __shared__ float s_lse2;
  if (hdr->status != 0) return;
  const int64_t row = blockIdx.x;
  const int tid = threadIdx.x;
  const T* z = Z + row * ld;
  T* g = dZ + row * ld_g;
  const float sc = softcap;
  const float inv_sc = CAP ? 1.f / softcap : 0.f;
  const int64_t head = ce_head(z, V);
  const int64_t nvec = (V - head) / VE;
  const int64_t tail0 = head + nvec * VE;
  const uint4* zv = reinterpret_cast<const uint4*>(z + head);
  // ---- pass 1: max and sum of exp2
  float m = -INFINITY, s = 0.f;
  for (int64_t j = tid; j < head + (V - tail0); j += kCeFusedThreads) {
    const int64_t col = j < head ? j : tail0 + (j - head);
    ce_merge(m, s, ce_u<CAP>(E::one(z + col), sc, inv_sc), 1.f);
  }
  for (int64_t v0 = tid; v0 < nvec; v0 += int64_t(kCeUnroll) * kCeFusedThreads) {
    uint4 raw[kCeUnroll];
#pragma unroll
    for (int u = 0; u < kCeUnroll; ++u) {
      const int64_t v = v0 + int64_t(u) * kCeFusedThreads;
      raw[u] = v < nvec ? __ldg(zv + v) : E::neg_inf();
    }
    float gz = -INFINITY;
#pragma unroll
    for (int u = 0; u < kCeUnroll; ++u) gz = fmaxf(gz, E::vmax(raw[u]));
    if (gz == -INFINITY) continue;
    const float mn = fmaxf(m, ce_u<CAP>(gz, sc, inv_sc));
    float a0 = 0.f, a1 = 0.f;
#pragma unroll
    for (int u = 0; u < kCeUnroll; ++u) {
      if (v0 + int64_t(u) * kCeFusedThreads >= nvec) break;
#pragma unroll
      for (int k = 0; k < VE; k += 2) {
        float d;
        a0 += ex2a(fmaf(capped<CAP>(E::get(raw[u], k), sc, inv_sc, &d), kLog2e, -mn));
        a1 += ex2a(fmaf(capped<CAP>(E::get(raw[u], k + 1), sc, inv_sc, &d), kLog2e, -mn));
      }
    }
    s = s * ex2a(m - mn) + (a0 + a1);
    m = mn;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
    const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
    ce_merge(m, s, m2, s2);
  }
  if ((tid & 31) == 0) {
    red_m[tid >> 5] = m;
    red_s[tid >> 5] = s;
  }
  __syncthreads();
  const int64_t lab = labels[row];
  const bool valid = lab != ignore_index;
  if (tid == 0) {
    float M = red_m[0], S = red_s[0];
    for (int w = 1; w < kW; ++w) ce_merge(M, S, red_m[w], red_s[w]);
    const float lse2 = M + log2f(S);
    const float l = lse2 * kLn2;
    float yt = 0.f;
    if (valid) {
      float d;
      yt = capped<CAP>(E::one(z + lab), sc, inv_sc, &d);
    }
    if (lse_out) lse_out[row] = l;
    row_loss[row] = valid ? l - yt : 0.f;
    s_lse2 = lse2;
  }
  __syncthreads();
  // ---- pass 2: the gradient, reading the row again (mostly from L2)
  const long long nv = hdr->n_valid;
  const float scale = (valid && nv > 0) ? dloss / float(nv) : 0.f;
  const float lse2 = scale != 0.f ? s_lse2 : 0.f;
  const bool same_phase = ce_head(g, V) == head;
  uint4* gv = reinterpret_cast<uint4*>(g + head);
  for (int64_t j = tid; j < head + (V - tail0); j += kCeFusedThreads) {
    const int64_t col = j < head ? j : tail0 + (j - head);
    E::store_one(g + col, scale != 0.f ? ce_grad<CAP>(E::one(z + col), sc, inv_sc, lse2, scale,
                                                      col == lab)
                                       : 0.f);
  }
  const int lab_rel = ce_lab_rel(lab, head, valid);
  for (int64_t v0 = tid; v0 < nvec; v0 += int64_t(kCeUnroll) * kCeFusedThreads) {
    uint4 raw[kCeUnroll];
#pragma unroll
    for (int u = 0; u < kCeUnroll; ++u) {
      const int64_t v = v0 + int64_t(u) * kCeFusedThreads;
      if (v < nvec) raw[u] = __ldcs(zv + v);
    }
#pragma unroll
    for (int u = 0; u < kCeUnroll; ++u) {
      const int64_t v = v0 + int64_t(u) * kCeFusedThreads;
      if (v >= nvec) break;
      float gg[VE];
      if (scale != 0.f) {
        ce_vec_grad<T, CAP>(raw[u], sc, inv_sc, lse2, scale, gg);
        ce_vec_label<T, CAP>(raw[u], lab_rel - int(v) * VE, sc, inv_sc, scale, gg);
      } else {
#pragma unroll
        for (int k = 0; k < VE; ++k) gg[k] = 0.f;
      }
      if (same_phase) {
        uint4 out;
#pragma unroll
        for (int k = 0; k < VE; k += 2) E::put(out, k, gg[k], gg[k + 1]);
        __stcs(gv + v, out);
      } else {
#pragma unroll
        for (int k = 0; k < VE; ++k) E::store_one(g + head + v * VE + k, gg[k]);
      }
    }
  }
}

}  // namespace flce

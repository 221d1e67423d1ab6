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

// G for one element: (exp(y - lse) - [label]) * dy/dz * scale.
template <bool CAP>
__device__ __forceinline__ float ce_grad(float z, float sc, float inv_sc, float lse2, float scale,
                                         bool is_label) {
  float d;
  const float y = capped<CAP>(z, sc, inv_sc, &d);
  const float p = ex2a(fmaf(y, kLog2e, -lse2));
  return (is_label ? p - 1.f : p) * (CAP ? d * scale : scale);
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
  const int64_t lab_rel = lab - head;  // label's position within the vector run
  for (int64_t v0 = tid; v0 < nvec; v0 += int64_t(kCeUnroll) * kCeThreads) {
    uint4 raw[kCeUnroll];
#pragma unroll
    for (int u = 0; u < kCeUnroll; ++u) {
      const int64_t v = v0 + int64_t(u) * kCeThreads;
      if (v < nvec) raw[u] = __ldcs(zv + v);
    }
#pragma unroll
    for (int u = 0; u < kCeUnroll; ++u) {
      const int64_t v = v0 + int64_t(u) * kCeThreads;
      if (v >= nvec) break;
      const int64_t rel = lab_rel - v * VE;  // in [0, VE) when the label is here
      uint4 out;
#pragma unroll
      for (int k = 0; k < VE; k += 2) {
        const float g0 = ce_grad<CAP>(E::get(raw[u], k), sc, inv_sc, lse2, scale, rel == k);
        const float g1 =
            ce_grad<CAP>(E::get(raw[u], k + 1), sc, inv_sc, lse2, scale, rel == k + 1);
        E::put(out, k, g0, g1);
      }
      __stcs(gv + v, out);
    }
  }
}

}  // namespace flce

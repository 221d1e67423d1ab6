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

namespace flce {

// Forward and backward in one pass over HBM, for a caller that holds the
// logits and wants the loss and the logit gradient together: one read and
// one write of each row instead of two reads and a write.
//
// ce_fused_pipe_kernel (rows up to kCeFusedRowMax bytes): a persistent block
// per SM keeps two row buffers in shared memory.  While it works on row k
// from one buffer -- the row's (max, sum-exp), its lse, then its gradient
// written to global memory -- one bulk asynchronous copy brings the 16-byte
// aligned interior of its next row into the other buffer, so the row reads
// and the gradient writes overlap.  The few elements before the first and
// after the last 16-byte boundary of a row go through plain loads, so every
// access stays inside the row.  Waits on the copies are bounded: a wait that
// gives up records FLCE_ERR_TIMEOUT, waits (bounded) for the copy still in
// flight and returns.
//
// ce_fused_rows_kernel (longer rows): one block per row, the row read twice
// (the second time mostly from L2, it was loaded moments before).  N_valid
// must be known (labels_kernel ran first); dloss is a host value.  dZ may be
// Z (in place).
constexpr int kCeFusedThreads = 512;
constexpr int kCeFusedRowMax = 112 * 1024;

template <typename T, bool CAP>
__global__ void __launch_bounds__(kCeFusedThreads, 1)
    ce_fused_pipe_kernel(const T* Z, int64_t ld, T* dZ, int64_t ld_g, int64_t BT, int64_t V,
                         const int64_t* __restrict__ labels, int64_t ignore_index,
                         float softcap, float dloss, float* __restrict__ lse_out,
                         float* __restrict__ row_loss, WsHeader* hdr, uint32_t buf_bytes,
                         unsigned long long wait_limit_ns) {
  using E = CeElem<T>;
  constexpr int VE = E::kVec;
  constexpr int kW = kCeFusedThreads / 32;
  extern __shared__ __align__(128) uint8_t s_buf[];
  __shared__ uint64_t full[2];
  __shared__ float red_m[kW], red_s[kW];
  __shared__ float s_lse2;
  if (hdr->status != 0) return;
  const int tid = threadIdx.x;
  const float sc = softcap;
  const float inv_sc = CAP ? 1.f / softcap : 0.f;
  const long long nv = hdr->n_valid;
  const uint64_t pol = policy_evict_first();
  if (tid == 0) {
    mbar_init(&full[0], 1);
    mbar_init(&full[1], 1);
    fence_barrier_init();
  }
  __syncthreads();
  // Row `row`'s aligned interior into buffer b (thread 0).
  auto issue = [&](int64_t row, int b) {
    const T* z = Z + row * ld;
    const int64_t head = ce_head(z, V);
    const uint32_t bytes = uint32_t(((V - head) / VE) * 16);
    fence_proxy_async_smem();  // the buffer's earlier generic reads come first
    if (bytes) {
      mbar_arrive_expect_tx(&full[b], bytes);
      bulk_load_g2s(s_buf + size_t(b) * buf_bytes, z + head, bytes, &full[b], pol);
    } else {
      mbar_arrive(&full[b]);
    }
  };
  int64_t row = blockIdx.x;
  if (tid == 0 && row < BT) issue(row, 0);
  bool failed = false;
  for (int64_t k = 0; row < BT; ++k, row += gridDim.x) {
    const int b = int(k & 1);
    const int64_t next = row + gridDim.x;
    if (tid == 0 && next < BT) issue(next, b ^ 1);  // freed at the end of iteration k - 1
    const bool got = mbar_wait_bounded(&full[b], uint32_t((k >> 1) & 1), wait_limit_ns, nullptr);
    if (!__syncthreads_and(got)) {
      failed = true;
      break;
    }
    const T* z = Z + row * ld;
    T* g = dZ + row * ld_g;
    const int64_t head = ce_head(z, V);
    const int64_t nvec = (V - head) / VE;
    const int64_t tail0 = head + nvec * VE;
    const uint4* sv = reinterpret_cast<const uint4*>(s_buf + size_t(b) * buf_bytes);
    // ---- the row's max and sum
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
        raw[u] = v < nvec ? sv[v] : E::neg_inf();
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
        for (int kk = 0; kk < VE; kk += 2) {
          float d;
          a0 += ex2a(fmaf(capped<CAP>(E::get(raw[u], kk), sc, inv_sc, &d), kLog2e, -mn));
          a1 += ex2a(fmaf(capped<CAP>(E::get(raw[u], kk + 1), sc, inv_sc, &d), kLog2e, -mn));
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
    // ---- the row's gradient, from the buffer
    const float scale = (valid && nv > 0) ? dloss / float(nv) : 0.f;
    const float lse2 = scale != 0.f ? s_lse2 : 0.f;
    const bool same_phase = ce_head(g, V) == head;
    uint4* gv = reinterpret_cast<uint4*>(g + head);
    for (int64_t j = tid; j < head + (V - tail0); j += kCeFusedThreads) {
      const int64_t col = j < head ? j : tail0 + (j - head);
      E::store_one(g + col, scale != 0.f ? ce_grad<CAP>(E::one(z + col), sc, inv_sc, lse2,
                                                        scale, col == lab)
                                         : 0.f);
    }
    const int64_t lab_rel = lab - head;
    for (int64_t v = tid; v < nvec; v += kCeFusedThreads) {
      const uint4 raw = sv[v];
      const int64_t rel = lab_rel - v * VE;
      float gg[VE];
#pragma unroll
      for (int kk = 0; kk < VE; ++kk)
        gg[kk] = scale != 0.f
                     ? ce_grad<CAP>(E::get(raw, kk), sc, inv_sc, lse2, scale, rel == kk)
                     : 0.f;
      if (same_phase) {
        uint4 out;
#pragma unroll
        for (int kk = 0; kk < VE; kk += 2) E::put(out, kk, gg[kk], gg[kk + 1]);
        __stcs(gv + v, out);
      } else {
#pragma unroll
        for (int kk = 0; kk < VE; ++kk) E::store_one(g + head + v * VE + kk, gg[kk]);
      }
    }
    __syncthreads();  // both buffers' readers are done before the next refill
  }
  if (failed && tid == 0) {
    atomicCAS(&hdr->status, 0, kStatusTimeout);
    // both buffers' copies may still be in flight: let them land
    const int64_t k = (row - int64_t(blockIdx.x)) / gridDim.x;
    mbar_wait_bounded(&full[k & 1], uint32_t((k >> 1) & 1), kDrainLimitNs, nullptr);
    if (row + gridDim.x < BT)
      mbar_wait_bounded(&full[(k + 1) & 1], uint32_t(((k + 1) >> 1) & 1), kDrainLimitNs,
                        nullptr);
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
  const int64_t lab_rel = lab - head;
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
      const int64_t rel = lab_rel - v * VE;
      float gg[VE];
#pragma unroll
      for (int k = 0; k < VE; ++k)
        gg[k] = scale != 0.f
                    ? ce_grad<CAP>(E::get(raw[u], k), sc, inv_sc, lse2, scale, rel == k)
                    : 0.f;
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

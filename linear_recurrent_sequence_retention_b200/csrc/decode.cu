// Single-token recurrent decode step (abeam.tech summary of Sun et al. 2023,
// section 「学習は並列、生成は状態更新」): per sequence n and head h,
//     S <- gamma_h S + k^T v     (in place),    o = q S.
//
// The float32 state [N, H, dk, dv] is the only large operand: each step reads
// and writes it once, so the kernel is bound by HBM bandwidth.  Layout of the
// work: a block owns 32*VEC consecutive columns of one (n, h) state and all
// dk rows; lane l streams the VEC-wide column group l of every row it owns
// (rows are 512 B apart for VEC=4, so every warp load is one fully used,
// contiguous 512-byte segment), warps take rows w, w+8, ...  Partial sums of
// q_i S'_ij over the rows are reduced across the 8 warps in shared memory.
// Loads/stores use streaming (evict-first) hints: the state is far larger than
// L2 and is not reused within a step.
#include "launch.h"

namespace ret {
namespace {

constexpr int kWarps = 8;
constexpr int kUnroll = 8;   // rows in flight per thread

template <int VEC> struct Vec;
template <> struct Vec<4> {
  using T = float4;
  static __device__ __forceinline__ T ld(const float* p) { return __ldcs(reinterpret_cast<const float4*>(p)); }
  static __device__ __forceinline__ void st(float* p, T x) { __stcs(reinterpret_cast<float4*>(p), x); }
  static __device__ __forceinline__ float get(const T& x, int i) {
    return i == 0 ? x.x : i == 1 ? x.y : i == 2 ? x.z : x.w;
  }
  static __device__ __forceinline__ void set(T& x, int i, float y) {
    if (i == 0) x.x = y; else if (i == 1) x.y = y; else if (i == 2) x.z = y; else x.w = y;
  }
};
template <> struct Vec<1> {
  using T = float;
  static __device__ __forceinline__ T ld(const float* p) { return __ldcs(p); }
  static __device__ __forceinline__ void st(float* p, T x) { __stcs(p, x); }
  static __device__ __forceinline__ float get(const T& x, int) { return x; }
  static __device__ __forceinline__ void set(T& x, int, float y) { x = y; }
};

template <typename Tin, typename To, int VEC>
__global__ void __launch_bounds__(kWarps * 32)
decode_step_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k,
                   const Tin* __restrict__ v, float* __restrict__ state, To* __restrict__ o,
                   int H, int dk, int dv, HeadDecay dec) {
  extern __shared__ float sm[];
  float* qs = sm;                 // [dk]
  float* ks = qs + dk;            // [dk]
  float* red = ks + dk;           // [kWarps][32*VEC]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int h = blockIdx.y, n = blockIdx.z;
  const size_t head = static_cast<size_t>(n) * H + h;
  const int col0 = (blockIdx.x * 32 + lane) * VEC;
  const bool colok = col0 < dv;   // VEC divides dv, so a group is all-in or all-out

  for (int i = threadIdx.x; i < dk; i += kWarps * 32) {
    qs[i] = Io<Tin>::ld(q, head * dk + i);
    ks[i] = Io<Tin>::ld(k, head * dk + i);
  }
  const float gam = dec.gamma[h];
  float vv[VEC];
#pragma unroll
  for (int e = 0; e < VEC; ++e) vv[e] = colok ? Io<Tin>::ld(v, head * dv + col0 + e) : 0.f;
  __syncthreads();

  float acc[VEC];
#pragma unroll
  for (int e = 0; e < VEC; ++e) acc[e] = 0.f;
  float* S = state + head * dk * dv;
  if (colok) {
    for (int i0 = warp; i0 < dk; i0 += kWarps * kUnroll) {
      typename Vec<VEC>::T x[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        int i = i0 + u * kWarps;
        if (i < dk) x[u] = Vec<VEC>::ld(S + static_cast<size_t>(i) * dv + col0);
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        int i = i0 + u * kWarps;
        if (i < dk) {
          const float ki = ks[i], qi = qs[i];
#pragma unroll
          for (int e = 0; e < VEC; ++e) {
            float s = fmaf(gam, Vec<VEC>::get(x[u], e), ki * vv[e]);
            Vec<VEC>::set(x[u], e, s);
            acc[e] = fmaf(qi, s, acc[e]);
          }
          Vec<VEC>::st(S + static_cast<size_t>(i) * dv + col0, x[u]);
        }
      }
    }
  }
#pragma unroll
  for (int e = 0; e < VEC; ++e) red[warp * 32 * VEC + lane * VEC + e] = acc[e];
  __syncthreads();
  for (int c = threadIdx.x; c < 32 * VEC; c += kWarps * 32) {
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) t += red[w * 32 * VEC + c];
    const int col = blockIdx.x * 32 * VEC + c;
    if (col < dv) Io<To>::st(o, head * dv + col, t);
  }
}

template <typename Tin, typename To, int VEC>
cudaError_t decode_typed(const void* q, const void* k, const void* v, float* state, void* o,
                         int N, int H, int dk, int dv, const HeadDecay& dec, cudaStream_t s) {
  size_t smem = sizeof(float) * (2 * dk + kWarps * 32 * VEC);
  auto kern = decode_step_kernel<Tin, To, VEC>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid((dv + 32 * VEC - 1) / (32 * VEC), H, N);
  kern<<<grid, kWarps * 32, smem, s>>>(static_cast<const Tin*>(q), static_cast<const Tin*>(k),
                                       static_cast<const Tin*>(v), state, static_cast<To*>(o),
                                       H, dk, dv, dec);
  return cudaGetLastError();
}

template <typename Tin, typename To>
cudaError_t decode_vec(const void* q, const void* k, const void* v, float* state, void* o,
                       int N, int H, int dk, int dv, const HeadDecay& dec, cudaStream_t s) {
  if (dv % 4 == 0) return decode_typed<Tin, To, 4>(q, k, v, state, o, N, H, dk, dv, dec, s);
  return decode_typed<Tin, To, 1>(q, k, v, state, o, N, H, dk, dv, dec, s);
}

}  // namespace

cudaError_t launch_decode_step(const void* q, const void* k, const void* v, DType in_t,
                               float* state, void* o, DType o_t, int N, int H, int dk, int dv,
                               const HeadDecay& dec, cudaStream_t s) {
  using bf = __nv_bfloat16;
  if (in_t == DType::F32)
    return o_t == DType::F32 ? decode_vec<float, float>(q, k, v, state, o, N, H, dk, dv, dec, s)
                             : decode_vec<float, bf>(q, k, v, state, o, N, H, dk, dv, dec, s);
  return o_t == DType::F32 ? decode_vec<bf, float>(q, k, v, state, o, N, H, dk, dv, dec, s)
                           : decode_vec<bf, bf>(q, k, v, state, o, N, H, dk, dv, dec, s);
}

}  // namespace ret

// Residual linear attention (RLA), the variant on the RAttention page (section
// "Residual Linear Attention (RLA) 수식"): a state without decay,
// S_t = S_(t-1) + phi(k_t)^T v_t, read w tokens late, o_t = phi(q_t) S_(t-w-1).
// With k''_t = phi(k_(t-w-1)) and v''_t = v_(t-w-1) (zero before the
// sequence) that is o_t = sum_{m <= t} (phi(q_t) . k''_m) v''_m, the retention
// of the other pages at gamma = 1, so the chunkwise forward kernels compute it
// after one pass that maps and shifts the inputs.  phi is the softmax over the
// head dimension (the page calls a softmax-based feature map the best choice
// and gives no formula).
#include "launch.h"

namespace ret {
namespace {

constexpr int kRlaWarps = 8;

template <typename T> __device__ __forceinline__ float ldf(const T* p, size_t i);
template <> __device__ __forceinline__ float ldf<float>(const float* p, size_t i) { return p[i]; }
template <> __device__ __forceinline__ float ldf<__nv_bfloat16>(const __nv_bfloat16* p, size_t i) {
  return __bfloat162float(p[i]);
}
template <typename T> __device__ __forceinline__ void stf(T* p, size_t i, float x);
template <> __device__ __forceinline__ void stf<float>(float* p, size_t i, float x) { p[i] = x; }
template <> __device__ __forceinline__ void stf<__nv_bfloat16>(__nv_bfloat16* p, size_t i, float x) {
  p[i] = __float2bfloat16_rn(x);
}

// Softmax of one row of d elements (one warp), written to out (or zeros).
template <typename T>
__device__ __forceinline__ void softmax_row(const T* in, T* out, int d, bool zero) {
  const int lane = threadIdx.x & 31;
  if (zero) {
    for (int j = lane; j < d; j += 32) stf<T>(out, j, 0.f);
    return;
  }
  float m = -INFINITY;
  for (int j = lane; j < d; j += 32) m = fmaxf(m, ldf<T>(in, j));
  for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float s = 0.f;
  for (int j = lane; j < d; j += 32) s += expf(ldf<T>(in, j) - m);
  for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  const float inv = 1.0f / s;
  for (int j = lane; j < d; j += 32) stf<T>(out, j, expf(ldf<T>(in, j) - m) * inv);
}

// VPL consecutive elements per lane as floats (one vector load / store).
template <typename T, int VPL> struct RowVec;
template <int VPL> struct RowVec<__nv_bfloat16, VPL> {
  static_assert(VPL == 2 || VPL == 4 || VPL == 8, "2, 4 or 8 bf16 per lane");
  static __device__ __forceinline__ void ld(const __nv_bfloat16* p, float (&x)[VPL]) {
    uint32_t w[VPL / 2];
    if constexpr (VPL == 2) {
      w[0] = *reinterpret_cast<const uint32_t*>(p);
    } else if constexpr (VPL == 4) {
      const uint2 u = *reinterpret_cast<const uint2*>(p);
      w[0] = u.x; w[1] = u.y;
    } else {
      const uint4 u = *reinterpret_cast<const uint4*>(p);
      w[0] = u.x; w[1] = u.y; w[2] = u.z; w[3] = u.w;
    }
#pragma unroll
    for (int i = 0; i < VPL / 2; ++i) {
      x[2 * i] = __uint_as_float(w[i] << 16);
      x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
  static __device__ __forceinline__ void st(__nv_bfloat16* p, const float (&x)[VPL]) {
    uint32_t w[VPL / 2];
#pragma unroll
    for (int i = 0; i < VPL / 2; ++i) {
      const __nv_bfloat162 b = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
      w[i] = *reinterpret_cast<const uint32_t*>(&b);
    }
    if constexpr (VPL == 2) {
      *reinterpret_cast<uint32_t*>(p) = w[0];
    } else if constexpr (VPL == 4) {
      *reinterpret_cast<uint2*>(p) = make_uint2(w[0], w[1]);
    } else {
      *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
};
template <int VPL> struct RowVec<float, VPL> {
  static_assert(VPL == 2 || VPL == 4 || VPL == 8, "2, 4 or 8 floats per lane");
  static __device__ __forceinline__ void ld(const float* p, float (&x)[VPL]) {
    if constexpr (VPL == 2) {
      const float2 u = *reinterpret_cast<const float2*>(p);
      x[0] = u.x; x[1] = u.y;
    } else {
#pragma unroll
      for (int i = 0; i < VPL / 4; ++i) {
        const float4 u = reinterpret_cast<const float4*>(p)[i];
        x[4 * i] = u.x; x[4 * i + 1] = u.y; x[4 * i + 2] = u.z; x[4 * i + 3] = u.w;
      }
    }
  }
  static __device__ __forceinline__ void st(float* p, const float (&x)[VPL]) {
    if constexpr (VPL == 2) {
      *reinterpret_cast<float2*>(p) = make_float2(x[0], x[1]);
    } else {
#pragma unroll
      for (int i = 0; i < VPL / 4; ++i)
        reinterpret_cast<float4*>(p)[i] = make_float4(x[4 * i], x[4 * i + 1], x[4 * i + 2], x[4 * i + 3]);
    }
  }
};

// Softmax of one row of 32 * VPL elements held in registers (one warp, one
// load and one store per lane).
template <typename T, int VPL>
__device__ __forceinline__ void softmax_row_reg(const T* in, T* out, bool zero) {
  const int lane = threadIdx.x & 31;
  float x[VPL];
  if (zero) {
#pragma unroll
    for (int i = 0; i < VPL; ++i) x[i] = 0.f;
    RowVec<T, VPL>::st(out + lane * VPL, x);
    return;
  }
  RowVec<T, VPL>::ld(in + lane * VPL, x);
  float m = x[0];
#pragma unroll
  for (int i = 1; i < VPL; ++i) m = fmaxf(m, x[i]);
  for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    x[i] = expf(x[i] - m);
    s += x[i];
  }
  for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  const float inv = 1.0f / s;
#pragma unroll
  for (int i = 0; i < VPL; ++i) x[i] *= inv;
  RowVec<T, VPL>::st(out + lane * VPL, x);
}

template <typename T>
__device__ __forceinline__ void softmax_any(const T* in, T* out, int d, bool zero) {
  switch (d) {
    case 64: softmax_row_reg<T, 2>(in, out, zero); break;
    case 128: softmax_row_reg<T, 4>(in, out, zero); break;
    case 256: softmax_row_reg<T, 8>(in, out, zero); break;
    default: softmax_row<T>(in, out, d, zero); break;
  }
}

// One warp per (token n, head h): q'[n] = phi(q[n]); k''[n] = phi(k[n-w-1]) and
// v''[n] = v[n-w-1] inside n's sequence, zero before it.  Rows of 64, 128 or
// 256 elements are held in registers (one vector load and store per lane);
// other widths take the strided loops.
template <typename T>
__global__ void __launch_bounds__(kRlaWarps * 32)
rla_inputs_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                  T* __restrict__ qf, T* __restrict__ ks, T* __restrict__ vs, SeqLayout L, int H,
                  int dk, int dv, int window) {
  const long long row = static_cast<long long>(blockIdx.x) * kRlaWarps + (threadIdx.x >> 5);
  if (row >= static_cast<long long>(L.Ttot) * H) return;
  const int n = static_cast<int>(row / H), h = static_cast<int>(row % H);
  int a = 0;
  if (L.cu == nullptr) {
    a = n - n % L.T;
  } else {
    int b;
    seq_bounds(L, seq_of_token(L, n), a, b);
    if (n < a || n >= b) a = n + 1;        // outside every sequence: no source token
  }
  const long long src = static_cast<long long>(n) - window - 1;
  const bool has = src >= a;
  const size_t qo = (static_cast<size_t>(n) * H + h) * dk;
  softmax_any<T>(q + qo, qf + qo, dk, false);
  const size_t ko = has ? (static_cast<size_t>(src) * H + h) * dk : 0;
  softmax_any<T>(k + ko, ks + qo, dk, !has);
  const int lane = threadIdx.x & 31;
  const size_t vo = (static_cast<size_t>(n) * H + h) * dv;
  const size_t vi = has ? (static_cast<size_t>(src) * H + h) * dv : 0;
  if ((dv * sizeof(T)) % 16 == 0) {
    // 16-byte copies: rows start 16-byte aligned when their byte length is a multiple of 16
    const int nvec = static_cast<int>(dv * sizeof(T) / 16);
    const uint4* sv = reinterpret_cast<const uint4*>(v + vi);
    uint4* dvp = reinterpret_cast<uint4*>(vs + vo);
    for (int j = lane; j < nvec; j += 32) dvp[j] = has ? sv[j] : make_uint4(0, 0, 0, 0);
  } else {
    for (int j = lane; j < dv; j += 32) stf<T>(vs, vo + j, has ? ldf<T>(v, vi + j) : 0.f);
  }
}

}  // namespace

cudaError_t launch_rla_inputs(const void* q, const void* k, const void* v, DType t, void* qf,
                              void* ks, void* vs, const SeqLayout& L, int H, int dk, int dv,
                              int window, cudaStream_t s) {
  if (L.Ttot == 0) return cudaSuccess;
  const long long rows = static_cast<long long>(L.Ttot) * H;
  const unsigned blocks = static_cast<unsigned>((rows + kRlaWarps - 1) / kRlaWarps);
  if (t == DType::F32)
    rla_inputs_kernel<float><<<blocks, kRlaWarps * 32, 0, s>>>(
        static_cast<const float*>(q), static_cast<const float*>(k), static_cast<const float*>(v),
        static_cast<float*>(qf), static_cast<float*>(ks), static_cast<float*>(vs), L, H, dk, dv,
        window);
  else
    rla_inputs_kernel<__nv_bfloat16><<<blocks, kRlaWarps * 32, 0, s>>>(
        static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
        static_cast<const __nv_bfloat16*>(v), static_cast<__nv_bfloat16*>(qf),
        static_cast<__nv_bfloat16*>(ks), static_cast<__nv_bfloat16*>(vs), L, H, dk, dv, window);
  return cudaGetLastError();
}

}  // namespace ret

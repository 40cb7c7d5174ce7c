// Rotary position encoding of q and k before retention.  The abeam.tech
// summary of Sun et al. 2023 (section 「Retentionは「内容に応じた参照」と「距離に
// よる忘却」を掛け合わせる」) rotates Q and K by position after the
// projections; the pages give no formula, and the standard rotary form is the
// one implemented: the pair (x[2i], x[2i+1]) of a token at position p (its
// index within its own sequence) turns by the angle p * theta_i with
// theta_i = base^(-2i/d).
//
// One streaming pass over q and k (HBM-bound; k may be absent).  One block per
// token; thread i owns pair i of every head, so the angle is computed once per
// (token, pair) and applied to 2H pairs.  The angle and the rotation come from
// the helpers in common.cuh (double-precision angle reduction, float32
// rotation); bf16 outputs are rounded to nearest once.
#include "launch.h"

namespace ret {
namespace {

template <typename T> struct Pair;
template <> struct Pair<float> {
  using V = float2;
  static __device__ __forceinline__ float2 ld(const float* p) { return *reinterpret_cast<const float2*>(p); }
  static __device__ __forceinline__ void st(float* p, float x, float y) {
    *reinterpret_cast<float2*>(p) = make_float2(x, y);
  }
  static __device__ __forceinline__ float lo(float2 v) { return v.x; }
  static __device__ __forceinline__ float hi(float2 v) { return v.y; }
};
template <> struct Pair<__nv_bfloat16> {
  using V = __nv_bfloat162;
  static __device__ __forceinline__ __nv_bfloat162 ld(const __nv_bfloat16* p) {
    return *reinterpret_cast<const __nv_bfloat162*>(p);
  }
  static __device__ __forceinline__ void st(__nv_bfloat16* p, float x, float y) {
    *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(x, y);
  }
  static __device__ __forceinline__ float lo(__nv_bfloat162 v) { return __low2float(v); }
  static __device__ __forceinline__ float hi(__nv_bfloat162 v) { return __high2float(v); }
};

template <typename T>
__global__ void __launch_bounds__(128)
rope_kernel(const T* __restrict__ q, const T* __restrict__ k, T* qo, T* ko, SeqLayout L, int H,
            int d, double log2_base) {
  const int n = blockIdx.x;
  if (n >= L.Ttot) return;
  int pos = 0;
  if (L.cu == nullptr) {
    pos = n % L.T;
  } else {
    const int s = seq_of_token(L, n);
    int a, b;
    seq_bounds(L, s, a, b);
    pos = (n >= a && n < b) ? n - a : 0;
  }
  const int half = d >> 1;
  for (int i = threadIdx.x; i < half; i += blockDim.x) {
    float sn, cs;
    rope_sincos(pos, rope_theta(i, d, log2_base), sn, cs);
    for (int h = 0; h < H; ++h) {
      const size_t off = (static_cast<size_t>(n) * H + h) * d + 2 * i;
      float y0, y1;
      const auto vq = Pair<T>::ld(q + off);
      rotate_pair(Pair<T>::lo(vq), Pair<T>::hi(vq), sn, cs, y0, y1);
      Pair<T>::st(qo + off, y0, y1);
      if (k != nullptr) {                  // k == nullptr: q alone
        const auto vk = Pair<T>::ld(k + off);
        rotate_pair(Pair<T>::lo(vk), Pair<T>::hi(vk), sn, cs, y0, y1);
        Pair<T>::st(ko + off, y0, y1);
      }
    }
  }
}

}  // namespace

cudaError_t launch_rope(const void* q, const void* k, DType t, void* qo, void* ko,
                        const SeqLayout& L, int H, int d, double base, cudaStream_t s) {
  if (L.Ttot == 0) return cudaSuccess;
  const int threads = d / 2 < 128 ? ((d / 2 + 31) / 32) * 32 : 128;
  const double lb = log2(base);
  if (t == DType::F32)
    rope_kernel<float><<<L.Ttot, threads, 0, s>>>(static_cast<const float*>(q),
                                                  static_cast<const float*>(k),
                                                  static_cast<float*>(qo), static_cast<float*>(ko),
                                                  L, H, d, lb);
  else
    rope_kernel<__nv_bfloat16><<<L.Ttot, threads, 0, s>>>(
        static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
        static_cast<__nv_bfloat16*>(qo), static_cast<__nv_bfloat16*>(ko), L, H, d, lb);
  return cudaGetLastError();
}

}  // namespace ret

// Rotary position encoding of q and k before retention.  The abeam.tech
// summary of Sun et al. 2023 (section 「Retentionは「内容に応じた参照」と「距離に
// よる忘却」を掛け合わせる」) rotates Q and K by position after the
// projections; the pages give no formula, and the standard rotary form is the
// one implemented: the pair (x[2i], x[2i+1]) of a token at position p (its
// index within its own sequence) turns by the angle p * theta_i with
// theta_i = base^(-2i/d).
//
// One streaming pass over q and k (HBM-bound).  One block per token; thread i
// owns pair i of every head of q and k, so the angle is computed once per
// (token, pair) and applied to 2H pairs.  The angle is formed and reduced
// modulo 2 pi in double precision and its sine and cosine are taken in float
// (sincosf on an argument in [-pi, pi]), so that large positions keep float
// accuracy; the rotation itself is float32, and bf16 outputs are rounded to
// nearest once.
#include "launch.h"

namespace ret {
namespace {

constexpr double kTwoPi = 6.283185307179586476925286766559;

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
    const double theta = exp2(-(2.0 * i / d) * log2_base);
    const double r = static_cast<double>(pos) * theta;
    const double turns = rint(r * (1.0 / kTwoPi));
    const float ang = static_cast<float>(fma(-turns, kTwoPi, r));
    float sn, cs;
    sincosf(ang, &sn, &cs);
    for (int h = 0; h < H; ++h) {
      const size_t off = (static_cast<size_t>(n) * H + h) * d + 2 * i;
      const auto vq = Pair<T>::ld(q + off);
      const auto vk = Pair<T>::ld(k + off);
      const float q0 = Pair<T>::lo(vq), q1 = Pair<T>::hi(vq);
      const float k0 = Pair<T>::lo(vk), k1 = Pair<T>::hi(vk);
      Pair<T>::st(qo + off, fmaf(q0, cs, -q1 * sn), fmaf(q0, sn, q1 * cs));
      Pair<T>::st(ko + off, fmaf(k0, cs, -k1 * sn), fmaf(k0, sn, k1 * cs));
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

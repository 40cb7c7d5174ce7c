// Standalone per-head GroupNorm + Swish gate (abeam.tech summary of Sun et al.
// 2023, section 「多時間尺度・ゲート・正規化で表現力を補う」; mlnews.online abstract
// page for arXiv 2307.08621, summary bullets: GroupNorm per head before the
// heads are concatenated):
//     y = ((o - mean) / sqrt(var + eps) * w + b) * g * sigmoid(g)
// with mean and biased variance over the dv channels of one (token, head).
// One warp per (token, head) row; the row stays in registers between the two
// statistics passes and the output pass, so o and g are read once.
#include "launch.h"

namespace ret {
namespace {

constexpr int kRowsPerBlock = 8;
constexpr int kMaxPerLane = 32;   // dv <= 1024

template <typename Ti, typename Tg, typename To>
__global__ void __launch_bounds__(kRowsPerBlock * 32)
norm_gate_kernel(const Ti* __restrict__ o, const Tg* __restrict__ g,
                 const float* __restrict__ w, const float* __restrict__ b, float eps,
                 To* __restrict__ y, long long nrows, int H, int dv) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const long long row = static_cast<long long>(blockIdx.x) * kRowsPerBlock + warp;
  if (row >= nrows) return;
  const int h = static_cast<int>(row % H);
  const size_t base = static_cast<size_t>(row) * dv;
  float x[kMaxPerLane];
  float s = 0.f;
#pragma unroll
  for (int e = 0; e < kMaxPerLane; ++e) {
    int c = lane + 32 * e;
    x[e] = c < dv ? Io<Ti>::ld(o, base + c) : 0.f;
    s += x[e];
  }
  for (int off = 16; off; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  const float mean = s / dv;
  float q = 0.f;
#pragma unroll
  for (int e = 0; e < kMaxPerLane; ++e) {
    int c = lane + 32 * e;
    if (c < dv) q += (x[e] - mean) * (x[e] - mean);
  }
  for (int off = 16; off; off >>= 1) q += __shfl_xor_sync(0xffffffffu, q, off);
  const float rstd = 1.0f / sqrtf(q / dv + eps);
#pragma unroll
  for (int e = 0; e < kMaxPerLane; ++e) {
    int c = lane + 32 * e;
    if (c < dv) {
      float t = (x[e] - mean) * rstd;
      if (w) t *= w[h * dv + c];
      if (b) t += b[h * dv + c];
      float gv = Io<Tg>::ld(g, base + c);
      Io<To>::st(y, base + c, t * (gv / (1.0f + expf(-gv))));
    }
  }
}

template <typename Ti, typename Tg, typename To>
cudaError_t ng_typed(const void* o, const void* g, const float* w, const float* b, float eps,
                     void* y, int ntok, int H, int dv, cudaStream_t s) {
  long long nrows = static_cast<long long>(ntok) * H;
  long long blocks = (nrows + kRowsPerBlock - 1) / kRowsPerBlock;
  if (blocks == 0) return cudaSuccess;
  norm_gate_kernel<Ti, Tg, To><<<static_cast<unsigned>(blocks), kRowsPerBlock * 32, 0, s>>>(
      static_cast<const Ti*>(o), static_cast<const Tg*>(g), w, b, eps, static_cast<To*>(y),
      nrows, H, dv);
  return cudaGetLastError();
}

template <typename Ti, typename Tg>
cudaError_t ng_out(const void* o, const void* g, const float* w, const float* b, float eps,
                   void* y, DType y_t, int ntok, int H, int dv, cudaStream_t s) {
  if (y_t == DType::F32) return ng_typed<Ti, Tg, float>(o, g, w, b, eps, y, ntok, H, dv, s);
  return ng_typed<Ti, Tg, __nv_bfloat16>(o, g, w, b, eps, y, ntok, H, dv, s);
}

template <typename Ti>
cudaError_t ng_gate(const void* o, const void* g, DType g_t, const float* w, const float* b,
                    float eps, void* y, DType y_t, int ntok, int H, int dv, cudaStream_t s) {
  if (g_t == DType::F32) return ng_out<Ti, float>(o, g, w, b, eps, y, y_t, ntok, H, dv, s);
  return ng_out<Ti, __nv_bfloat16>(o, g, w, b, eps, y, y_t, ntok, H, dv, s);
}

}  // namespace

cudaError_t launch_norm_gate(const void* o, DType o_t, const void* g, DType g_t,
                             const float* w, const float* b, float eps, void* y, DType y_t,
                             int ntok, int H, int dv, cudaStream_t s) {
  if (o_t == DType::F32) return ng_gate<float>(o, g, g_t, w, b, eps, y, y_t, ntok, H, dv, s);
  return ng_gate<__nv_bfloat16>(o, g, g_t, w, b, eps, y, y_t, ntok, H, dv, s);
}

}  // namespace ret

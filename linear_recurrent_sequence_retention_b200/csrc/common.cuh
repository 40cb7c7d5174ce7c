// Shared device helpers of libretention: dtype access, per-head decay powers,
// the device error word and the sequence/chunk bookkeeping used by every
// chunkwise kernel.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace ret {

constexpr int kMaxHeads = 64;

// Bits of the per-device error word (see retention_check_device_error).
constexpr unsigned kErrTimeout = 1u;     // a bounded wait gave up
constexpr unsigned kErrDeviceData = 2u;  // cu_seqlens inconsistent
constexpr unsigned kErrRange = 4u;       // a value exceeded the fp16 range of the tensor-core operands

// Per-head decay constants, computed on the host in double precision from the
// caller's gamma and passed by value.  gamma^n is evaluated as
// exp2(n * log2(gamma)) for one integer n at a time (never as gamma^i *
// gamma^-j, which overflows for small gamma); gamma == 0 is kept exact
// (0^0 = 1, 0^n = 0 for n > 0).
struct HeadDecay {
  float gamma[kMaxHeads];        // gamma_h rounded to float
  float log2g[kMaxHeads];
  unsigned long long zero_mask;  // bit h set when gamma_h == 0
};

__device__ __forceinline__ float gpow(const HeadDecay& d, int h, int n) {
  if (n == 0) return 1.0f;
  if ((d.zero_mask >> h) & 1ull) return 0.0f;
  return exp2f(static_cast<float>(n) * d.log2g[h]);
}

// The same power for one head whose constants are already in registers.
struct Decay1 {
  float log2g;
  bool zero;
  __device__ __forceinline__ Decay1(const HeadDecay& d, int h)
      : log2g(d.log2g[h]), zero(((d.zero_mask >> h) & 1ull) != 0) {}
  __device__ __forceinline__ float pow(int n) const {
    if (n == 0) return 1.0f;
    if (zero) return 0.0f;
    return exp2f(static_cast<float>(n) * log2g);
  }
};

// ---- dtype access --------------------------------------------------------

template <typename T> struct Io;
template <> struct Io<float> {
  static __device__ __forceinline__ float ld(const float* p, size_t i) { return p[i]; }
  static __device__ __forceinline__ void st(float* p, size_t i, float x) { p[i] = x; }
};
template <> struct Io<__nv_bfloat16> {
  static __device__ __forceinline__ float ld(const __nv_bfloat16* p, size_t i) {
    return __bfloat162float(p[i]);
  }
  static __device__ __forceinline__ void st(__nv_bfloat16* p, size_t i, float x) {
    p[i] = __float2bfloat16_rn(x);
  }
};

__device__ __forceinline__ void raise_error(unsigned* err, unsigned bits) {
  if (err) atomicOr(err, bits);
}

// ---- rotary position encoding ------------------------------------------------
//
// The standard rotary form (the pages name a position rotation of Q and K but
// give no formula): the pair (x[2i], x[2i+1]) of a token at position p turns
// by p * theta_i, theta_i = base^(-2i/d).  theta_i is passed in double; the
// angle is formed and reduced modulo 2 pi in double precision and its sine and
// cosine are taken in float on an argument in [-pi, pi], so that large
// positions keep float accuracy.  Every kernel that rotates uses this helper
// and rotate_pair, so the rotated values agree bit for bit between them.
__device__ __forceinline__ double rope_theta(int i, int d, double log2_base) {
  return exp2(-(2.0 * i / d) * log2_base);
}
__device__ __forceinline__ void rope_sincos(int pos, double theta, float& sn, float& cs) {
  constexpr double kTwoPi = 6.283185307179586476925286766559;
  const double r = static_cast<double>(pos) * theta;
  const double turns = rint(r * (1.0 / kTwoPi));
  const float ang = static_cast<float>(fma(-turns, kTwoPi, r));
  sincosf(ang, &sn, &cs);
}
// (x0, x1) rotated by the angle whose sine and cosine are sn, cs (float32).
__device__ __forceinline__ void rotate_pair(float x0, float x1, float sn, float cs, float& y0,
                                            float& y1) {
  y0 = fmaf(x0, cs, -x1 * sn);
  y1 = fmaf(x0, sn, x1 * cs);
}

// ---- sequences and chunks -------------------------------------------------
//
// Both layouts are handled as packed sequences over a flat token axis of
// length Ttot: the padded layout [B, T, ...] is the packed layout with
// offsets 0, T, 2T, ..., so token t of sequence b has flat index b*T + t.
struct SeqLayout {
  const int32_t* cu;      // device offsets [nseq+1], or nullptr (padded)
  int nseq;               // number of sequences (B when padded)
  int T;                  // tokens per sequence when padded
  int Ttot;               // total flat tokens
  int chunk;              // chunk length
  long long nslots;       // workspace state slots; every slot index is checked
                          // against it, so malformed offsets stay in bounds
};

// [begin, end) of sequence s on the flat token axis, clamped to [0, Ttot]
// and made non-decreasing, so that a malformed cu_seqlens can never cause an
// out-of-bounds access (the prep kernel reports it).
__device__ __forceinline__ void seq_bounds(const SeqLayout& L, int s, int& a, int& b) {
  if (L.cu == nullptr) {
    a = s * L.T;
    b = a + L.T;
    return;
  }
  a = L.cu[s];
  b = L.cu[s + 1];
  a = a < 0 ? 0 : (a > L.Ttot ? L.Ttot : a);
  b = b < a ? a : (b > L.Ttot ? L.Ttot : b);
}

// Sequence that owns flat token n (largest s with begin(s) <= n).
__device__ __forceinline__ int seq_of_token(const SeqLayout& L, int n) {
  if (L.cu == nullptr) return n / L.T;
  int lo = 0, hi = L.nseq - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    int a = L.cu[mid];
    if (a <= n) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

}  // namespace ret

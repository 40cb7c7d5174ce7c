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

// ---------------------------------------------------------------------------
// Several tokens per sequence in one pass over the state.  For tokens
// t = 0..Tn-1 entering with state S (the recurrence above, unrolled):
//     o_t = gamma^(t+1) q_t S + sum_{j<=t} gamma^(t-j) (q_t . k_j) v_j
//     S'  = gamma^Tn S + sum_j gamma^(Tn-1-j) k_j^T v_j
// so the state is read and written once for all Tn tokens.  A block owns up to
// 512 columns of one (n, h) state: warp w the 64 columns 64w.., two per lane,
// over all dk rows, so a warp's output sums need no other warp.  Every thread
// walks groups of 4 rows (the next group's loads in flight while this one is
// folded in), folds each row into its Tn output partial sums and updates it in
// place.  q_t, k_j (with their decay factors), the block's v columns and the
// small Tn x Tn score block live in shared memory.
// ---------------------------------------------------------------------------
constexpr int kMultiCols = 512;                 // columns per block
constexpr int kMultiWarpCols = 64;              // columns per warp (2 per lane)

// Four consecutive elements as floats (8-byte aligned bf16, 16-byte aligned f32).
__device__ __forceinline__ float4 ld4(const __nv_bfloat16* p) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u),
                     __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u));
}
__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }

template <typename Tin, typename To, int MAXT>
__global__ void __launch_bounds__(kWarps * 32)
decode_multi_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k,
                    const Tin* __restrict__ v, float* __restrict__ state, To* __restrict__ o,
                    int Tn, int H, int dk, int dv, HeadDecay dec) {
  extern __shared__ __align__(16) float sm[];
  float* qf = sm;                          // [MAXT][dk]  q_t, then q_t gamma^(t+1)
  float* kw = qf + MAXT * dk;              // [MAXT][dk]  k_j, then k_j gamma^(Tn-1-j)
  float* vs = kw + MAXT * dk;              // [MAXT][512] v_j of this block's columns
  float* A = vs + MAXT * kMultiCols;       // [MAXT][MAXT] (q_t . k_j) gamma^(t-j), j <= t
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int h = blockIdx.y, n = blockIdx.z;
  const int cblk = blockIdx.x * kMultiCols;
  const int ncols = min(kMultiCols, dv - cblk);
  const int wc = warp * kMultiWarpCols + lane * 2;     // this thread's first column in the block
  const bool colok = wc < ncols;                       // 4 divides dv, so both columns are in
  const Decay1 dg(dec, h);

  // q, k of all tokens and v of this block's columns into shared memory
  for (int idx4 = threadIdx.x * 4; idx4 < MAXT * dk; idx4 += kWarps * 32 * 4) {
    const int t = idx4 / dk, i = idx4 % dk;
    float4 aq = make_float4(0.f, 0.f, 0.f, 0.f), ak = aq;
    if (t < Tn) {
      const size_t row = (static_cast<size_t>(n) * Tn + t) * H + h;
      aq = ld4(q + row * dk + i);
      ak = ld4(k + row * dk + i);
    }
    *reinterpret_cast<float4*>(qf + idx4) = aq;
    *reinterpret_cast<float4*>(kw + idx4) = ak;
  }
  for (int idx4 = threadIdx.x * 4; idx4 < MAXT * kMultiCols; idx4 += kWarps * 32 * 4) {
    const int t = idx4 / kMultiCols, c = idx4 % kMultiCols;
    float4 av = make_float4(0.f, 0.f, 0.f, 0.f);
    if (t < Tn && c < ncols) av = ld4(v + ((static_cast<size_t>(n) * Tn + t) * H + h) * dv + cblk + c);
    *reinterpret_cast<float4*>(vs + idx4) = av;
  }
  __syncthreads();
  for (int idx = warp; idx < MAXT * MAXT; idx += kWarps) {   // one (t, j) per warp
    const int t = idx / MAXT, j = idx % MAXT;
    float a = 0.f;
    if (j <= t && t < Tn) {
      for (int i = lane; i < dk; i += 32) a = fmaf(qf[t * dk + i], kw[j * dk + i], a);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
      a *= dg.pow(t - j);
    }
    if (lane == 0) A[idx] = a;
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < MAXT * dk; idx += kWarps * 32) {
    const int t = idx / dk;
    qf[idx] *= dg.pow(t + 1);
    kw[idx] *= t < Tn ? dg.pow(Tn - 1 - t) : 0.f;
  }
  __syncthreads();
  if (!colok) return;

  float acc[MAXT][2];
#pragma unroll
  for (int t = 0; t < MAXT; ++t) acc[t][0] = acc[t][1] = 0.f;
  const float gT = dg.pow(Tn);
  float* S = state + (static_cast<size_t>(n) * H + h) * dk * dv + cblk + wc;
  // rows g0..g0+3 per iteration; the next group's rows are already in flight
  // while this group is folded in
  float2 xn[4];
#pragma unroll
  for (int r = 0; r < 4; ++r) xn[r] = __ldcs(reinterpret_cast<const float2*>(S + static_cast<size_t>(r) * dv));
  for (int g0 = 0; g0 < dk; g0 += 4) {
    float2 x[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) x[r] = xn[r];
    if (g0 + 4 < dk) {
#pragma unroll
      for (int r = 0; r < 4; ++r)
        xn[r] = __ldcs(reinterpret_cast<const float2*>(S + static_cast<size_t>(g0 + 4 + r) * dv));
    }
#pragma unroll
    for (int t = 0; t < MAXT; ++t) {
      const float4 qa = *reinterpret_cast<const float4*>(qf + t * dk + g0);
      const float qr[4] = {qa.x, qa.y, qa.z, qa.w};
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        acc[t][0] = fmaf(qr[r], x[r].x, acc[t][0]);
        acc[t][1] = fmaf(qr[r], x[r].y, acc[t][1]);
      }
    }
    float2 y[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) y[r] = make_float2(gT * x[r].x, gT * x[r].y);
#pragma unroll
    for (int j = 0; j < MAXT; ++j) {
      const float4 ka = *reinterpret_cast<const float4*>(kw + j * dk + g0);
      const float2 vj = *reinterpret_cast<const float2*>(vs + j * kMultiCols + wc);
      const float kr[4] = {ka.x, ka.y, ka.z, ka.w};
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        y[r].x = fmaf(kr[r], vj.x, y[r].x);
        y[r].y = fmaf(kr[r], vj.y, y[r].y);
      }
    }
#pragma unroll
    for (int r = 0; r < 4; ++r)
      __stcs(reinterpret_cast<float2*>(S + static_cast<size_t>(g0 + r) * dv), y[r]);
  }
  // o_t = (gamma^(t+1) q_t S) + sum_{j<=t} A[t][j] v_j for this thread's two columns
#pragma unroll
  for (int t = 0; t < MAXT; ++t) {
    if (t >= Tn) break;
    float s0 = acc[t][0], s1 = acc[t][1];
    for (int j = 0; j <= t; ++j) {
      const float2 vj = *reinterpret_cast<const float2*>(vs + j * kMultiCols + wc);
      s0 = fmaf(A[t * MAXT + j], vj.x, s0);
      s1 = fmaf(A[t * MAXT + j], vj.y, s1);
    }
    const size_t ob = ((static_cast<size_t>(n) * Tn + t) * H + h) * dv + cblk + wc;
    Io<To>::st(o, ob, s0);
    Io<To>::st(o, ob + 1, s1);
  }
}

template <typename Tin, typename To, int MAXT>
cudaError_t decode_multi_typed(const void* q, const void* k, const void* v, float* state,
                               void* o, int N, int Tn, int H, int dk, int dv,
                               const HeadDecay& dec, cudaStream_t s) {
  const size_t smem = sizeof(float) * (2 * MAXT * dk + MAXT * kMultiCols + MAXT * MAXT);
  auto kern = decode_multi_kernel<Tin, To, MAXT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid((dv + kMultiCols - 1) / kMultiCols, H, N);
  kern<<<grid, kWarps * 32, smem, s>>>(static_cast<const Tin*>(q), static_cast<const Tin*>(k),
                                       static_cast<const Tin*>(v), state, static_cast<To*>(o),
                                       Tn, H, dk, dv, dec);
  return cudaGetLastError();
}

template <typename Tin, typename To>
cudaError_t decode_multi(const void* q, const void* k, const void* v, float* state, void* o,
                         int N, int Tn, int H, int dk, int dv, const HeadDecay& dec,
                         cudaStream_t s) {
  if (Tn <= 4) return decode_multi_typed<Tin, To, 4>(q, k, v, state, o, N, Tn, H, dk, dv, dec, s);
  if (Tn <= 8) return decode_multi_typed<Tin, To, 8>(q, k, v, state, o, N, Tn, H, dk, dv, dec, s);
  return decode_multi_typed<Tin, To, 16>(q, k, v, state, o, N, Tn, H, dk, dv, dec, s);
}

}  // namespace

cudaError_t launch_decode_steps(const void* q, const void* k, const void* v, DType in_t,
                                float* state, void* o, DType o_t, int N, int Tn, int H, int dk,
                                int dv, const HeadDecay& dec, unsigned* err, cudaStream_t s) {
  using bf = __nv_bfloat16;
  if (in_t == DType::BF16 && decode_steps_tc_preferred(Tn, dk, dv)) {
    // cudaErrorNotSupported: the tensor-core kernel declined before launching
    // anything (sizes past its index or tensor-map range); the CUDA-core one runs
    const cudaError_t e = launch_decode_steps_tc(q, k, v, state, o, o_t, N, Tn, H, dk, dv, dec, err, s);
    if (e != cudaErrorNotSupported) return e;
  }
  if (in_t == DType::F32)
    return o_t == DType::F32 ? decode_multi<float, float>(q, k, v, state, o, N, Tn, H, dk, dv, dec, s)
                             : decode_multi<float, bf>(q, k, v, state, o, N, Tn, H, dk, dv, dec, s);
  return o_t == DType::F32 ? decode_multi<bf, float>(q, k, v, state, o, N, Tn, H, dk, dv, dec, s)
                           : decode_multi<bf, bf>(q, k, v, state, o, N, Tn, H, dk, dv, dec, s);
}

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

// Backward of the chunkwise form on the tensor-core forward kernels (bf16
// inputs).  The gradients of the pages' retention (abeam.tech summary of Sun et
// al. 2023, 「学習は並列、生成は状態更新」 and 「長文の学習にはチャンク再帰を使う」)
// are three retentions of the same kind as the forward, with the operand roles
// exchanged:
//     dq_n = sum_{m<=n} gamma^(n-m) (dO_n . v_m) k_m + gamma^(n+1) dO_n S0^T
//          = causal(q = dO, k = V, v = K, state in = S0^T)
//     dv_m = sum_{n>=m} gamma^(n-m) (k_m . q_n) dO_n + gamma^(T-1-m) k_m dS_T
//          = anti-causal(q = K, k = Q, v = dO, state in = dS_T)
//     dk_m = sum_{n>=m} gamma^(n-m) (v_m . dO_n) q_n + gamma^(T-1-m) v_m dS_T^T
//          = anti-causal(q = V, k = dO, v = Q, state in = dS_T^T)
//     dS0  = sum_n gamma^(n+1) q_n^T dO_n + gamma^T dS_T
//          = the final state of the anti-causal (Q, dO) pass.
// The dK pass's state, sum gamma^(j+1) dO_j^T q_j, is the transpose of the dV
// pass's: it runs no state pass of its own and reads the dV pass's state slots
// transposed (K-major), with an fp16 copy of Q as its value operand.
// The anti-causal retention walks the chunks last to first carrying the state
// of everything after each chunk, F_(c-1) = gamma^L F_c + sum_j gamma^(j+1)
// k_j^T v_j, and reads it as gamma^(L-1-i) q_i F_c; started from dS_T it
// gives the final-state terms above, and its last state is dS0 exactly (every
// gamma, 0 included: 0^0 = 1).  With d_v = 512 the two retentions whose score
// contracts over d_v (dQ: dO . v, dK: v . dO) exceed the forward kernels'
// 256-wide query rows; the score is linear in that contraction, so each runs
// as two passes over the d_v halves, the second adding its result to the
// first's (float32 outputs):
//     dq = causal(dO[:, :256], V[:, :256], K) + causal(dO[:, 256:], V[:, 256:], K)
// with the states entering split by rows the same way, and likewise for dK.
// This file holds the two small kernels that composition needs (the d_v
// halves of v and dO, the state transposes) and the host sequence of
// launches; the retentions themselves run in chunkwise_tc.cu.
#include "launch.h"

namespace ret {
namespace {

constexpr int kCopyThreads = 256;
constexpr int kCopyTok = 8;          // tokens per block
constexpr int kCopyIlp = 4;          // 16-byte loads in flight per thread

// dst0/dst1[n][h][:] = the two halves of head h of token row n of src; a half
// is `hvec` 16-byte vectors.  A block moves kCopyTok consecutive rows; each
// thread issues kCopyIlp loads before its stores.
__global__ void __launch_bounds__(kCopyThreads)
split_heads_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst0,
                   uint4* __restrict__ dst1, int ntok, int H, int hvec) {
  const int n0 = blockIdx.x * kCopyTok;
  const int row_vec = 2 * H * hvec;
  const int rows = min(kCopyTok, ntok - n0);
  const int total = rows * row_vec;
  for (int base = threadIdx.x; base < total; base += kCopyIlp * kCopyThreads) {
    uint4 v[kCopyIlp];
#pragma unroll
    for (int u = 0; u < kCopyIlp; ++u) {
      const int e = base + u * kCopyThreads;
      if (e < total) v[u] = src[static_cast<size_t>(n0) * row_vec + e];
    }
#pragma unroll
    for (int u = 0; u < kCopyIlp; ++u) {
      const int e = base + u * kCopyThreads;
      if (e >= total) continue;
      const int n = n0 + e / row_vec, w = e % row_vec;
      const int h = w / (2 * hvec), half = (w / hvec) & 1, x = w % hvec;
      (half ? dst1 : dst0)[(static_cast<size_t>(n) * H + h) * hvec + x] = v[u];
    }
  }
}

// out[s][h] = in[s][h]^T  (in: [dk][dv] -> out: [dv][dk]), 32 x 32 tiles.  The
// rows of out are split in two arrays at row hd (hd = dv: out0 only): rows
// [0, hd) go to out0 [nseq*H][hd][dk], rows [hd, dv) to out1 likewise.
__global__ void transpose_states_kernel(const float* __restrict__ in, float* __restrict__ out0,
                                        float* __restrict__ out1, int dk, int dv, int hd) {
  __shared__ float tile[32][33];
  const size_t mat = static_cast<size_t>(blockIdx.z) * dk * dv;
  const int r0 = blockIdx.y * 32, c0 = blockIdx.x * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int r = r0 + i, c = c0 + threadIdx.x;
    tile[i][threadIdx.x] = (r < dk && c < dv) ? in[mat + static_cast<size_t>(r) * dv + c] : 0.f;
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int c = c0 + i, r = r0 + threadIdx.x;
    if (c < dv && r < dk) {
      const int half = c >= hd ? 1 : 0;
      float* out = half ? out1 : out0;
      out[(static_cast<size_t>(blockIdx.z) * hd + (c - half * hd)) * dk + r] = tile[threadIdx.x][i];
    }
  }
}

// Heads with 0 < gamma < kSmallGamma: the initial-state gradient
//     dS0 = sum_n gamma^(n+1) q_n^T dO_n + gamma^T dS_T
// again, in float32, over the tokens whose weight is still nonzero.  The
// anti-causal pass forms it from fp16 operands zeta_j k_j with zeta_j =
// gamma^(j+1), which for such gamma fall below fp16's normal range, while this
// sum is made of exactly those terms.  One block per (sequence, head).
constexpr float kSmallGamma = 1e-3f;

__global__ void small_gamma_state_kernel(const __nv_bfloat16* __restrict__ q,
                                         const __nv_bfloat16* __restrict__ d_out,
                                         const float* __restrict__ dS, float* __restrict__ dS0,
                                         SeqLayout L, int H, int dk, int dv, HeadDecay dec) {
  const int s = blockIdx.x, h = blockIdx.y;
  const float g = dec.gamma[h];
  if (!(g > 0.f && g < kSmallGamma)) return;
  int a, b;
  seq_bounds(L, s, a, b);
  // weights gamma^(n+1) that are still nonzero in float32 (a few tokens)
  constexpr int kMaxTok = 32;
  __shared__ float w[kMaxTok];
  __shared__ int nt;
  if (threadIdx.x == 0) {
    float x = g;
    int n = 0;
    while (n < kMaxTok && n < b - a && x > 0.f) {
      w[n] = x;
      x *= g;
      ++n;
    }
    nt = n;
  }
  __syncthreads();
  const int len = b - a;
  const float gT = len == 0 ? 1.f : gpow(dec, h, len);
  const size_t mat = (static_cast<size_t>(s) * H + h) * dk * dv;
  for (int e = threadIdx.x; e < dk * dv; e += blockDim.x) {
    const int i = e / dv, c = e % dv;
    float acc = dS ? gT * dS[mat + e] : 0.f;
    for (int n = 0; n < nt; ++n) {
      const size_t row = static_cast<size_t>(a + n) * H + h;
      acc = fmaf(w[n] * __bfloat162float(q[row * dk + i]), __bfloat162float(d_out[row * dv + c]), acc);
    }
    dS0[mat + e] = acc;
  }
}

// bf16 [ntok][H][2*hd] -> two [ntok][H][hd] arrays
cudaError_t split_halves(const void* src, void* dst0, void* dst1, int ntok, int H, int hd,
                         cudaStream_t s) {
  if (ntok == 0) return cudaSuccess;
  split_heads_kernel<<<(ntok + kCopyTok - 1) / kCopyTok, kCopyThreads, 0, s>>>(
      static_cast<const uint4*>(src), static_cast<uint4*>(dst0), static_cast<uint4*>(dst1), ntok,
      H, hd * 2 / 16);
  return cudaGetLastError();
}

cudaError_t transpose_split(const float* in, float* out0, float* out1, int nmat, int dk, int dv,
                            int hd, cudaStream_t s) {
  dim3 grid((dv + 31) / 32, (dk + 31) / 32, static_cast<unsigned>(nmat));
  transpose_states_kernel<<<grid, dim3(32, 8), 0, s>>>(in, out0, out1, dk, dv, hd);
  return cudaGetLastError();
}

}  // namespace

size_t chunkwise_bwd_tc_scratch_bytes(const SeqLayout& L, int H, int dk, int dv) {
  const size_t T = static_cast<size_t>(L.Ttot);
  auto r256 = [](size_t b) { return (b + 255) / 256 * 256; };
  const size_t st = r256(static_cast<size_t>(L.nseq) * H * dk * dv * 4);
  size_t b = st;                                         // S0^T (split in d_v halves)
  if (dv > 256) b += 4 * r256(T * H * (dv / 2) * 2);     // the d_v halves of dO and V
  return b;
}

cudaError_t launch_chunkwise_bwd_tc(const void* q, const void* k, const void* v,
                                    const void* d_out, const SeqLayout& L, const float* state_in,
                                    const float* d_state_out, float* dq, float* dk, float* dv,
                                    float* d_state_in, ChunkWorkspace ws, void* scratch, int H,
                                    int dk_, int dv_, const HeadDecay& dec, unsigned* err,
                                    cudaStream_t s) {
  const size_t T = static_cast<size_t>(L.Ttot);
  auto r256 = [](size_t b) { return (b + 255) / 256 * 256; };
  // d_v = 512: the passes contracting over d_v run on its two halves
  const bool split = dv_ > 256;
  const int hd = split ? dv_ / 2 : dv_;
  const int nh = split ? 2 : 1;
  char* p = static_cast<char*>(scratch);
  const size_t st_bytes = r256(static_cast<size_t>(L.nseq) * H * dk_ * dv_ * 4);
  float* s0t = reinterpret_cast<float*>(p); p += st_bytes;   // S0^T   [dv][dk] (split: 2 x [hd][dk])
  const size_t half_st = static_cast<size_t>(L.nseq) * H * hd * dk_;   // floats per half
  float* s0t_h[2] = {s0t, s0t + half_st};
  const void* doh[2] = {d_out, nullptr};
  const void* vh[2] = {v, nullptr};
  cudaError_t e = cudaSuccess;
  if (split) {
    const size_t half_in = r256(T * H * hd * 2);
    void* b0 = p; p += half_in;
    void* b1 = p; p += half_in;
    void* b2 = p; p += half_in;
    void* b3 = p;
    doh[0] = b0; doh[1] = b1; vh[0] = b2; vh[1] = b3;
    e = split_halves(d_out, b0, b1, L.Ttot, H, hd, s);
    if (e == cudaSuccess) e = split_halves(v, b2, b3, L.Ttot, H, hd, s);
  }
  const int nmat = L.nseq * H;
  if (e == cudaSuccess && state_in)
    e = transpose_split(state_in, s0t_h[0], s0t_h[1], nmat, dk_, dv_, hd, s);
  if (e != cudaSuccess) return e;
  const DType F = DType::F32;
  const bool ds = d_state_out != nullptr;
  // dQ: causal(q = dO, k = V, v = K) from S0^T (per d_v half, summed)
  for (int i = 0; i < nh && e == cudaSuccess; ++i)
    e = launch_chunkwise_tc(3, doh[i], vh[i], k, L, state_in ? s0t_h[i] : nullptr,
                            state_in != nullptr, nullptr, dq, F, nullptr, F, nullptr, nullptr, 0.f,
                            false, ws, H, hd, dk_, dec, err, s, i > 0, false);
  // dV: anti-causal(q = K, k = Q, v = dO) from dS_T; its final state is dS0
  if (e == cudaSuccess)
    e = launch_chunkwise_tc(3, k, q, d_out, L, d_state_out, ds, d_state_in, dv, F, nullptr, F,
                            nullptr, nullptr, 0.f, false, ws, H, dk_, dv_, dec, err, s, false,
                            true);
  if (e == cudaSuccess && d_state_in) {
    bool small = false;
    for (int h = 0; h < H; ++h) small = small || (dec.gamma[h] > 0.f && dec.gamma[h] < kSmallGamma);
    if (small) {
      small_gamma_state_kernel<<<dim3(static_cast<unsigned>(L.nseq), H), 256, 0, s>>>(
          static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(d_out),
          d_state_out, d_state_in, L, H, dk_, dv_, dec);
      e = cudaGetLastError();
    }
  }
  // dK: anti-causal(q = V, k = dO, v = Q) on the dV pass's states read
  // transposed (they start from dS_T, so the last chunk reads dS_T^T), its value
  // operand the fp16 copy of Q; per d_v half, summed
  if (e == cudaSuccess) e = launch_to_f16(q, ws.v16, static_cast<long long>(T) * H * dk_, err, s);
  for (int i = 0; i < nh && e == cudaSuccess; ++i) {
    StateRead sr;
    sr.transposed = true;
    sr.col0 = i * hd;
    sr.stored_dv = dv_;
    e = launch_chunkwise_tc(2, vh[i], doh[i], q, L, nullptr, ds, nullptr, dk, F, nullptr, F,
                            nullptr, nullptr, 0.f, false, ws, H, hd, dk_, dec, err, s, i > 0, true,
                            sr);
  }
  return e;
}

}  // namespace ret

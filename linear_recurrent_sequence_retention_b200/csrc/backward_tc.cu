// Backward of the chunkwise form on the tensor-core forward kernels (bf16
// inputs).  The gradients of the pages' retention (abeam.tech summary of Sun et
// al. 2023, 「学習は並列、生成は状態更新」 and 「長文の学習にはチャンク再帰を使う」)
// are three retentions of the same kind as the forward, with the operand roles
// exchanged:
//     dq_n = sum_{m<=n} gamma^(n-m) (dO_n . v_m) k_m + gamma^(n+1) dO_n S0^T
//          = forward(q = dO, k = V, v = K, state_in = S0^T)
//     dv_m = sum_{n>=m} gamma^(n-m) (k_m . q_n) dO_n
//          = forward(q = K, k = Q, v = dO) on every sequence read backwards
//     dk_m = sum_{n>=m} gamma^(n-m) (v_m . dO_n) q_n
//          = forward(q = V, k = dO, v = Q) on every sequence read backwards
//     dS0  = sum_n gamma^(n+1) q_n^T dO_n
//          = gamma * (final state of the backwards (k = Q, v = dO) pass)
// A final-state gradient dS_T adds gamma^(T-1-m) k_m dS_T to dv_m and
// gamma^(T-1-m) v_m dS_T^T to dk_m: at the backwards position m' = T-1-m that
// is gamma^(m') k dS_T, which the forward's read of an initial state,
// gamma^(m'+1) q S_in, gives with S_in = dS_T / gamma (and its transpose for
// dK); the backwards pass's final state then also carries gamma^(T-1) dS_T, so
// dS0 = gamma * final still holds.  Heads with gamma = 0 take S_in = 0 and a
// fix-up of the last token of each sequence (the only term left, gamma^0).
// (reading a sequence backwards turns "n >= m" into "n' <= m'" with the same
// distance).  With d_v = 512 the two passes whose score contracts over d_v
// (dQ: dO . v, dK: v . dO) exceed the forward kernels' 256-wide query rows;
// the score is linear in that contraction, so each runs as two passes over the
// d_v halves, the second adding its result to the first's (float32 outputs):
//     dq = forward(dO[:, :256], V[:, :256], K) + forward(dO[:, 256:], V[:, 256:], K)
// with the initial state's transpose split the same way, and likewise for dK.  This file holds the three small streaming kernels the
// composition needs (reverse the tokens of every sequence, transpose the
// initial state, scale the state gradient per head) and the host sequence of
// launches; the retentions themselves run in chunkwise_tc.cu.
#include "launch.h"

namespace ret {
namespace {

constexpr int kFlipThreads = 256;
constexpr int kFlipTok = 8;          // tokens per block
constexpr int kFlipIlp = 4;          // 16-byte loads in flight per thread

// dst[a + j] = src[b - 1 - j] for every sequence [a, b) of the flat token
// axis; a token row is `row_vec` 16-byte vectors.  A block moves kFlipTok
// consecutive destination rows; each thread issues kFlipIlp loads before its
// stores, so enough bytes are in flight to keep HBM busy.  Rows outside every
// sequence are left as they are.
__global__ void __launch_bounds__(kFlipThreads)
flip_tokens_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, SeqLayout L,
                   int row_vec) {
  __shared__ int srow[kFlipTok];
  const int n0 = blockIdx.x * kFlipTok;
  if (threadIdx.x < kFlipTok) {
    const int n = n0 + static_cast<int>(threadIdx.x);
    int m = -1;
    if (n < L.Ttot) {
      int a, b;
      seq_bounds(L, seq_of_token(L, n), a, b);
      if (n >= a && n < b) m = a + b - 1 - n;
    }
    srow[threadIdx.x] = m;
  }
  __syncthreads();
  const int total = kFlipTok * row_vec;
  for (int base = threadIdx.x; base < total; base += kFlipIlp * kFlipThreads) {
    uint4 v[kFlipIlp];
    int m[kFlipIlp], e[kFlipIlp];
#pragma unroll
    for (int u = 0; u < kFlipIlp; ++u) {
      e[u] = base + u * kFlipThreads;
      m[u] = e[u] < total ? srow[e[u] / row_vec] : -1;
      if (m[u] >= 0) v[u] = src[static_cast<size_t>(m[u]) * row_vec + e[u] % row_vec];
    }
#pragma unroll
    for (int u = 0; u < kFlipIlp; ++u)
      if (m[u] >= 0) dst[static_cast<size_t>(n0) * row_vec + e[u]] = v[u];
  }
}

// dst0/dst1[n][h][:] = the two halves of head h of token row m of src, where
// m = a + b - 1 - n (flip) or n, for every token n of a sequence [a, b); a
// half is `hvec` 16-byte vectors.  Same block shape as flip_tokens_kernel.
__global__ void __launch_bounds__(kFlipThreads)
split_heads_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst0,
                   uint4* __restrict__ dst1, SeqLayout L, int H, int hvec, int flip) {
  __shared__ int srow[kFlipTok];
  const int n0 = blockIdx.x * kFlipTok;
  if (threadIdx.x < kFlipTok) {
    const int n = n0 + static_cast<int>(threadIdx.x);
    int m = -1;
    if (n < L.Ttot) {
      int a, b;
      seq_bounds(L, seq_of_token(L, n), a, b);
      if (n >= a && n < b) m = flip ? a + b - 1 - n : n;
    }
    srow[threadIdx.x] = m;
  }
  __syncthreads();
  const int row_vec = 2 * H * hvec;
  const int total = kFlipTok * row_vec;
  for (int base = threadIdx.x; base < total; base += kFlipIlp * kFlipThreads) {
    uint4 v[kFlipIlp];
    int m[kFlipIlp], e[kFlipIlp];
#pragma unroll
    for (int u = 0; u < kFlipIlp; ++u) {
      e[u] = base + u * kFlipThreads;
      m[u] = e[u] < total ? srow[e[u] / row_vec] : -1;
      if (m[u] >= 0) v[u] = src[static_cast<size_t>(m[u]) * row_vec + e[u] % row_vec];
    }
#pragma unroll
    for (int u = 0; u < kFlipIlp; ++u) {
      if (m[u] < 0) continue;
      const int n = n0 + e[u] / row_vec, w = e[u] % row_vec;
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

// out[s][h] = x[s][h] / gamma_h (zero where gamma_h = 0) over [nseq*H][dk*dv].
__global__ void state_over_gamma_kernel(const float* __restrict__ x, float* __restrict__ out, int H,
                                        size_t per, HeadDecay dec) {
  const int mat = blockIdx.y;
  const float gm = dec.gamma[mat % H];
  const float inv = gm > 0.f ? 1.0f / gm : 0.f;
  const float* a = x + static_cast<size_t>(mat) * per;
  float* b = out + static_cast<size_t>(mat) * per;
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < per;
       i += static_cast<size_t>(gridDim.x) * blockDim.x)
    b[i] = a[i] * inv;
}

// Heads with gamma = 0: the final-state gradient reaches only the last token of
// each sequence, dv += k dS_T and dk += dS_T v (and an empty sequence passes it
// to d_state_in).  One block per (sequence, head).
__global__ void zero_gamma_fixup_kernel(const __nv_bfloat16* __restrict__ k,
                                        const __nv_bfloat16* __restrict__ v,
                                        const float* __restrict__ dS, float* __restrict__ dk,
                                        float* __restrict__ dv, float* __restrict__ d_state_in,
                                        SeqLayout L, int H, int dk_, int dv_, HeadDecay dec) {
  const int s = blockIdx.x, h = blockIdx.y;
  if (!((dec.zero_mask >> h) & 1ull)) return;
  int a, b;
  seq_bounds(L, s, a, b);
  const float* M = dS + (static_cast<size_t>(s) * H + h) * dk_ * dv_;
  if (b == a) {
    if (d_state_in) {
      float* out = d_state_in + (static_cast<size_t>(s) * H + h) * dk_ * dv_;
      for (int i = threadIdx.x; i < dk_ * dv_; i += blockDim.x) out[i] = M[i];
    }
    return;
  }
  const size_t last = static_cast<size_t>(b - 1) * H + h;
  for (int c = threadIdx.x; c < dv_; c += blockDim.x) {
    float x = 0.f;
    for (int i = 0; i < dk_; ++i) x = fmaf(__bfloat162float(k[last * dk_ + i]), M[static_cast<size_t>(i) * dv_ + c], x);
    dv[last * dv_ + c] += x;
  }
  for (int i = threadIdx.x; i < dk_; i += blockDim.x) {
    float x = 0.f;
    for (int c = 0; c < dv_; ++c) x = fmaf(M[static_cast<size_t>(i) * dv_ + c], __bfloat162float(v[last * dv_ + c]), x);
    dk[last * dk_ + i] += x;
  }
}

// x[s][h] *= gamma_h over [nmat = nseq*H][dk*dv].
__global__ void scale_states_kernel(float* __restrict__ x, int H, size_t per, HeadDecay dec) {
  const int mat = blockIdx.y;
  const float gm = dec.gamma[mat % H];
  float* p = x + static_cast<size_t>(mat) * per;
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < per;
       i += static_cast<size_t>(gridDim.x) * blockDim.x)
    p[i] *= gm;
}

cudaError_t flip(const void* src, void* dst, const SeqLayout& L, size_t row_bytes, cudaStream_t s) {
  if (L.Ttot == 0) return cudaSuccess;
  flip_tokens_kernel<<<(L.Ttot + kFlipTok - 1) / kFlipTok, kFlipThreads, 0, s>>>(
      static_cast<const uint4*>(src), static_cast<uint4*>(dst), L, static_cast<int>(row_bytes / 16));
  return cudaGetLastError();
}

// bf16 [Ttot][H][2*hd] -> two [Ttot][H][hd] arrays, optionally read backwards
cudaError_t split_halves(const void* src, void* dst0, void* dst1, const SeqLayout& L, int H, int hd,
                         bool reverse, cudaStream_t s) {
  if (L.Ttot == 0) return cudaSuccess;
  split_heads_kernel<<<(L.Ttot + kFlipTok - 1) / kFlipTok, kFlipThreads, 0, s>>>(
      static_cast<const uint4*>(src), static_cast<uint4*>(dst0), static_cast<uint4*>(dst1), L, H,
      hd * 2 / 16, reverse ? 1 : 0);
  return cudaGetLastError();
}

}  // namespace

size_t chunkwise_bwd_tc_scratch_bytes(const SeqLayout& L, int H, int dk, int dv) {
  const size_t T = static_cast<size_t>(L.Ttot);
  auto r256 = [](size_t b) { return (b + 255) / 256 * 256; };
  const size_t st = r256(static_cast<size_t>(L.nseq) * H * dk * dv * 4);
  size_t b = 2 * r256(T * H * dk * 2) + 2 * r256(T * H * dv * 2)  // q, k, v, dO read backwards
             + r256(T * H * dk * 4) + r256(T * H * dv * 4)         // dK, dV of the backwards passes
             + 3 * st;                                             // S0^T, dS_T / gamma and its transpose
  if (dv > 256)                                                    // d_v halves: dO, V forwards and
    b += 3 * r256(T * H * dv * 2) + 3 * 256;                       // dO backwards (+ split padding)
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
  char* p = static_cast<char*>(scratch);
  void* q_r = p;  p += r256(T * H * dk_ * 2);
  void* k_r = p;  p += r256(T * H * dk_ * 2);
  void* v_r = p;  p += r256(T * H * dv_ * 2);                 // split: its two halves
  void* do_r = p; p += r256(T * H * dv_ * 2);
  float* dk_r = reinterpret_cast<float*>(p); p += r256(T * H * dk_ * 4);
  float* dv_r = reinterpret_cast<float*>(p); p += r256(T * H * dv_ * 4);
  const size_t st_bytes = r256(static_cast<size_t>(L.nseq) * H * dk_ * dv_ * 4);
  float* s0t = reinterpret_cast<float*>(p); p += st_bytes;   // S0^T        [dv][dk] (split: 2 x [hd][dk])
  float* sv = reinterpret_cast<float*>(p);  p += st_bytes;   // dS_T / gamma [dk][dv]
  float* svt = reinterpret_cast<float*>(p); p += st_bytes;   // its transpose, split like S0^T
  const size_t half_st = static_cast<size_t>(L.nseq) * H * hd * dk_;   // floats per half
  const size_t half_in = r256(T * H * hd * 2);
  void* vh_r[2] = {v_r, static_cast<char*>(v_r) + half_in};
  void *doh_r[2] = {nullptr, nullptr}, *doh[2] = {nullptr, nullptr}, *vh[2] = {nullptr, nullptr};
  if (split) {
    doh_r[0] = p; p += half_in; doh_r[1] = p; p += half_in;
    doh[0] = p;   p += half_in; doh[1] = p;   p += half_in;
    vh[0] = p;    p += half_in; vh[1] = p;    p += half_in;
  }
  const size_t rq = static_cast<size_t>(H) * dk_ * 2, rv = static_cast<size_t>(H) * dv_ * 2;
  cudaError_t e = flip(q, q_r, L, rq, s);
  if (e == cudaSuccess) e = flip(k, k_r, L, rq, s);
  if (e == cudaSuccess) e = flip(d_out, do_r, L, rv, s);
  if (split) {
    if (e == cudaSuccess) e = split_halves(v, vh_r[0], vh_r[1], L, H, hd, true, s);
    if (e == cudaSuccess) e = split_halves(d_out, doh_r[0], doh_r[1], L, H, hd, true, s);
    if (e == cudaSuccess) e = split_halves(d_out, doh[0], doh[1], L, H, hd, false, s);
    if (e == cudaSuccess) e = split_halves(v, vh[0], vh[1], L, H, hd, false, s);
  } else if (e == cudaSuccess) {
    e = flip(v, v_r, L, rv, s);
  }
  float* s0t_h[2] = {s0t, s0t + half_st};
  float* svt_h[2] = {svt, svt + half_st};
  if (e == cudaSuccess && state_in) {
    dim3 grid((dv_ + 31) / 32, (dk_ + 31) / 32, static_cast<unsigned>(L.nseq) * H);
    transpose_states_kernel<<<grid, dim3(32, 8), 0, s>>>(state_in, s0t_h[0], s0t_h[1], dk_, dv_, hd);
    e = cudaGetLastError();
  }
  const size_t per = static_cast<size_t>(dk_) * dv_;
  if (e == cudaSuccess && d_state_out) {
    dim3 grid(static_cast<unsigned>((per + 1023) / 1024), static_cast<unsigned>(L.nseq) * H);
    state_over_gamma_kernel<<<grid, 256, 0, s>>>(d_state_out, sv, H, per, dec);
    e = cudaGetLastError();
    if (e == cudaSuccess) {
      dim3 tg((dv_ + 31) / 32, (dk_ + 31) / 32, static_cast<unsigned>(L.nseq) * H);
      transpose_states_kernel<<<tg, dim3(32, 8), 0, s>>>(sv, svt_h[0], svt_h[1], dk_, dv_, hd);
      e = cudaGetLastError();
    }
  }
  if (e != cudaSuccess) return e;
  const DType F = DType::F32;
  const bool ds = d_state_out != nullptr;
  const int nh = split ? 2 : 1;
  // dQ: forward(q = dO, k = V, v = K) from S0^T (per d_v half, summed)
  for (int i = 0; i < nh && e == cudaSuccess; ++i)
    e = launch_chunkwise_tc(3, split ? doh[i] : d_out, split ? vh[i] : v, k, L,
                            state_in ? s0t_h[i] : nullptr, state_in != nullptr, nullptr, dq, F,
                            nullptr, F, nullptr, nullptr, 0.f, false, ws, H, hd, dk_, dec, err, s,
                            i > 0);
  // dV on the sequences read backwards: forward(q = K, k = Q, v = dO); its final
  // state is sum_n gamma^n q_n^T dO_n, the initial-state gradient before one gamma
  if (e == cudaSuccess)
    e = launch_chunkwise_tc(3, k_r, q_r, do_r, L, ds ? sv : nullptr, ds, d_state_in, dv_r, F,
                            nullptr, F, nullptr, nullptr, 0.f, false, ws, H, dk_, dv_, dec, err, s);
  // dK on the sequences read backwards: forward(q = V, k = dO, v = Q) (per d_v half, summed)
  for (int i = 0; i < nh && e == cudaSuccess; ++i)
    e = launch_chunkwise_tc(3, vh_r[i], split ? doh_r[i] : do_r, q_r, L, ds ? svt_h[i] : nullptr,
                            ds, nullptr, dk_r, F, nullptr, F, nullptr, nullptr, 0.f, false, ws, H,
                            hd, dk_, dec, err, s, i > 0);
  if (e == cudaSuccess) e = flip(dv_r, dv, L, static_cast<size_t>(H) * dv_ * 4, s);
  if (e == cudaSuccess) e = flip(dk_r, dk, L, static_cast<size_t>(H) * dk_ * 4, s);
  if (e == cudaSuccess && d_state_in) {
    dim3 grid(static_cast<unsigned>((per + 1023) / 1024), static_cast<unsigned>(L.nseq) * H);
    scale_states_kernel<<<grid, 256, 0, s>>>(d_state_in, H, per, dec);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess && ds && dec.zero_mask) {
    zero_gamma_fixup_kernel<<<dim3(static_cast<unsigned>(L.nseq), H), 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v), d_state_out,
        dk, dv, d_state_in, L, H, dk_, dv_, dec);
    e = cudaGetLastError();
  }
  return e;
}

}  // namespace ret

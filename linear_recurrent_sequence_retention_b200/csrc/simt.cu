// CUDA-core (FFMA) kernels of libretention: the parallel form, and the
// chunkwise form for float32 inputs (where tensor cores have no float32 mode
// and parity at 1e-5 relative needs float32 products).
//
// Parallel form (abeam.tech summary of Sun et al. 2023, section
// 「学習は並列、生成は状態更新」): O = (Q K^T * D) V with D_nm = gamma^(n-m),
// n >= m.  Chunkwise form (same page, 「長文の学習にはチャンク再帰を使う」):
// inside a chunk the parallel form, across chunks a decayed read of the state
// carried from the previous chunk; the state is updated at each chunk end.
#include "launch.h"

namespace ret {
namespace {

constexpr int kRows = 16;     // query rows per block
constexpr int kKeys = 16;     // keys per tile
constexpr int kThreads = 256;

// ---------------------------------------------------------------------------
// Parallel form: block = (16 query rows, head h, batch b); thread t owns
// output column t for all 16 rows.  Scores are formed 16 x 16 at a time and
// weighted by gamma^(n-m) for m <= n.
// ---------------------------------------------------------------------------
template <typename Tin, typename To>
__global__ void __launch_bounds__(kThreads)
parallel_simt_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k,
                     const Tin* __restrict__ v, To* __restrict__ o,
                     int T, int H, int dk, int dv, HeadDecay dec) {
  extern __shared__ float smem[];
  const int ldq = dk + 1;
  float* qs = smem;                      // [kRows][dk+1]
  float* ks = qs + kRows * ldq;          // [kKeys][dk+1]
  float* vs = ks + kKeys * ldq;          // [kKeys][dv]
  float* ss = vs + kKeys * dv;           // [kRows][kKeys+1]

  const int n0 = blockIdx.x * kRows, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x;
  const size_t tok0 = static_cast<size_t>(b) * T;

  for (int e = tid; e < kRows * dk; e += kThreads) {
    int r = e / dk, d = e % dk, n = n0 + r;
    qs[r * ldq + d] = n < T ? Io<Tin>::ld(q, ((tok0 + n) * H + h) * dk + d) : 0.f;
  }
  float acc[kRows];
#pragma unroll
  for (int r = 0; r < kRows; ++r) acc[r] = 0.f;

  const int last_row = min(n0 + kRows, T) - 1;
  for (int m0 = 0; m0 <= last_row; m0 += kKeys) {
    __syncthreads();
    for (int e = tid; e < kKeys * dk; e += kThreads) {
      int c = e / dk, d = e % dk, m = m0 + c;
      ks[c * ldq + d] = m < T ? Io<Tin>::ld(k, ((tok0 + m) * H + h) * dk + d) : 0.f;
    }
    for (int e = tid; e < kKeys * dv; e += kThreads) {
      int c = e / dv, d = e % dv, m = m0 + c;
      vs[c * dv + d] = m < T ? Io<Tin>::ld(v, ((tok0 + m) * H + h) * dv + d) : 0.f;
    }
    __syncthreads();
    {
      int r = tid / kKeys, c = tid % kKeys;
      int n = n0 + r, m = m0 + c;
      float s = 0.f;
      for (int d = 0; d < dk; ++d) s = fmaf(qs[r * ldq + d], ks[c * ldq + d], s);
      ss[r * (kKeys + 1) + c] = (m <= n && n < T) ? s * gpow(dec, h, n - m) : 0.f;
    }
    __syncthreads();
    if (tid < dv) {
#pragma unroll
      for (int r = 0; r < kRows; ++r) {
        float a = acc[r];
        for (int c = 0; c < kKeys; ++c) a = fmaf(ss[r * (kKeys + 1) + c], vs[c * dv + tid], a);
        acc[r] = a;
      }
    }
  }
  for (int col = tid; col < dv; col += kThreads) {
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      int n = n0 + r;
      if (n < T) Io<To>::st(o, ((tok0 + n) * H + h) * dv + col, acc[r]);
    }
  }
}

// ---------------------------------------------------------------------------
// Chunk bookkeeping for packed sequences: chunk_base[s] = number of chunks of
// all sequences before s.  One block; also checks cu_seqlens.
// ---------------------------------------------------------------------------
//
// order[0..nseq) lists the sequences by chunk count, longest first (ties in any
// order; counts of kOrderBins-1 chunks or more share the top bin), so that a
// grid walking sequences in that order starts the longest serial chains first.
constexpr int kOrderBins = 2048;

__global__ void chunk_prep_kernel(SeqLayout L, int32_t* chunk_base, int32_t* order, unsigned* err) {
  __shared__ int carry;
  __shared__ int bad;
  __shared__ int bins[kOrderBins];
  if (threadIdx.x == 0) { carry = 0; bad = 0; }
  for (int i = threadIdx.x; i < kOrderBins; i += blockDim.x) bins[i] = 0;
  __syncthreads();
  if (threadIdx.x == 0) {
    if (L.cu[0] != 0 || L.cu[L.nseq] != L.Ttot) bad = 1;
  }
  for (int base = 0; base < L.nseq; base += blockDim.x) {
    int s = base + threadIdx.x;
    int n = 0;
    if (s < L.nseq) {
      int a0 = L.cu[s], b0 = L.cu[s + 1];
      if (b0 < a0) atomicOr(&bad, 1);
      int a, b;
      seq_bounds(L, s, a, b);
      n = ceil_div(b - a, L.chunk);
    }
    // inclusive scan over the block (Hillis-Steele through shared memory)
    __shared__ int sc[1024];
    sc[threadIdx.x] = n;
    __syncthreads();
    for (int off = 1; off < blockDim.x; off <<= 1) {
      int x = threadIdx.x >= off ? sc[threadIdx.x - off] : 0;
      __syncthreads();
      sc[threadIdx.x] += x;
      __syncthreads();
    }
    if (s < L.nseq) {
      chunk_base[s] = carry + sc[threadIdx.x] - n;
      atomicAdd(&bins[min(n, kOrderBins - 1)], 1);
    }
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) carry += sc[threadIdx.x];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    chunk_base[L.nseq] = carry;
    if (bad) raise_error(err, kErrDeviceData);
  }
  // bins -> first position of each chunk count in the longest-first order:
  // exclusive scan from the top bin down (two bins per thread)
  __shared__ int pos[kOrderBins];
  {
    const int hi = kOrderBins - 1 - 2 * threadIdx.x;      // this thread's bins: hi, hi-1
    const int c0 = hi >= 0 ? bins[hi] : 0, c1 = hi >= 1 ? bins[hi - 1] : 0;
    __shared__ int ps[1024];
    ps[threadIdx.x] = c0 + c1;
    __syncthreads();
    for (int off = 1; off < blockDim.x; off <<= 1) {
      int x = threadIdx.x >= off ? ps[threadIdx.x - off] : 0;
      __syncthreads();
      ps[threadIdx.x] += x;
      __syncthreads();
    }
    const int before = ps[threadIdx.x] - (c0 + c1);          // sequences in higher bins
    if (hi >= 0) pos[hi] = before;
    if (hi >= 1) pos[hi - 1] = before + c0;
  }
  __syncthreads();
  for (int s = threadIdx.x; s < L.nseq; s += blockDim.x) {
    int a, b;
    seq_bounds(L, s, a, b);
    const int n = ceil_div(b - a, L.chunk);
    order[atomicAdd(&pos[min(n, kOrderBins - 1)], 1)] = s;
  }
}

__device__ __forceinline__ long long slot_of(const SeqLayout& L, const int32_t* chunk_base,
                                             int s, int c) {
  if (L.cu == nullptr) return static_cast<long long>(s) * ceil_div(L.T, L.chunk) + c;
  return static_cast<long long>(chunk_base[s]) + c;
}

// ---------------------------------------------------------------------------
// Chunkwise state pass: block = (32 state columns, head h, sequence s).
// Walks the sequence's chunks in order; before each chunk it stores the state
// entering it (S_prev) in the workspace, then applies
//     S <- gamma^L S + sum_j gamma^(L-1-j) k_j^T v_j.
// With kRev the chunks are walked from the last to the first and the update is
//     F <- gamma^L F + sum_j gamma^(j+1) k_j^T v_j
// (the backward's state of the future, called with k = q and v = dO): the
// value stored for chunk c is then the state of everything after it.
// Lane = column, warp w owns state rows w, w+8, ... (dk <= 256 -> 32 rows).
// ---------------------------------------------------------------------------
constexpr int kStateTok = 32;

template <typename Tin, bool kRev>
__global__ void __launch_bounds__(kThreads)
chunk_state_simt_kernel(const Tin* __restrict__ k, const Tin* __restrict__ v, SeqLayout L,
                        const int32_t* __restrict__ chunk_base,
                        const float* __restrict__ state_in, float* __restrict__ state_out,
                        float* __restrict__ ws_states, int H, int dk, int dv, HeadDecay dec) {
  extern __shared__ float smem[];
  float* kt = smem;                      // [kStateTok][dk]
  float* vt = kt + kStateTok * dk;       // [kStateTok][32]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int col = blockIdx.x * 32 + lane;
  const int h = blockIdx.y, s = blockIdx.z;
  const bool colok = col < dv;
  int a, b;
  seq_bounds(L, s, a, b);
  const int len = b - a;

  float S[32];
#pragma unroll
  for (int r = 0; r < 32; ++r) {
    int i = warp + 8 * r;
    S[r] = (state_in && colok && i < dk)
               ? state_in[((static_cast<size_t>(s) * H + h) * dk + i) * dv + col] : 0.f;
  }
  const int nch = ceil_div(len, L.chunk);
  for (int cc = 0; cc < nch; ++cc) {
    const int c = kRev ? nch - 1 - cc : cc;
    const long long slot = slot_of(L, chunk_base, s, c);
    if (slot >= 0 && slot < L.nslots) {
      float* dst = ws_states + (static_cast<size_t>(slot) * H + h) * dk * dv;
#pragma unroll
      for (int r = 0; r < 32; ++r) {
        int i = warp + 8 * r;
        if (colok && i < dk) dst[static_cast<size_t>(i) * dv + col] = S[r];
      }
    }
    const int c0 = a + c * L.chunk;
    const int Lc = min(L.chunk, b - c0);
    const float gL = gpow(dec, h, Lc);
#pragma unroll
    for (int r = 0; r < 32; ++r) S[r] *= gL;
    for (int j0 = 0; j0 < Lc; j0 += kStateTok) {
      __syncthreads();
      for (int e = threadIdx.x; e < kStateTok * dk; e += kThreads) {
        int jj = e / dk, d = e % dk, j = j0 + jj;
        kt[e] = j < Lc ? Io<Tin>::ld(k, (static_cast<size_t>(c0 + j) * H + h) * dk + d) : 0.f;
      }
      for (int e = threadIdx.x; e < kStateTok * 32; e += kThreads) {
        int jj = e / 32, cc = e % 32, j = j0 + jj, cl = blockIdx.x * 32 + cc;
        vt[e] = (j < Lc && cl < dv)
                    ? gpow(dec, h, kRev ? j + 1 : Lc - 1 - j) *
                          Io<Tin>::ld(v, (static_cast<size_t>(c0 + j) * H + h) * dv + cl)
                    : 0.f;
      }
      __syncthreads();
      const int jn = min(kStateTok, Lc - j0);
      for (int jj = 0; jj < jn; ++jj) {
        const float vz = vt[jj * 32 + lane];
#pragma unroll
        for (int r = 0; r < 32; ++r) {
          int i = warp + 8 * r;
          if (i < dk) S[r] = fmaf(kt[jj * dk + i], vz, S[r]);
        }
      }
    }
  }
  if (state_out && colok) {
#pragma unroll
    for (int r = 0; r < 32; ++r) {
      int i = warp + 8 * r;
      if (i < dk) state_out[((static_cast<size_t>(s) * H + h) * dk + i) * dv + col] = S[r];
    }
  }
}

// ---------------------------------------------------------------------------
// Chunkwise output pass: block = (16 flat token rows, head h).  Every row n
// finds its sequence, its chunk start cs and the slot of the state entering
// that chunk, then
//     o_n = sum_{cs <= m <= n} gamma^(n-m) (q_n.k_m) v_m + gamma^(n-cs+1) q_n S_prev.
// Thread t owns column t (dv <= 256).  With `gated`, the per-head GroupNorm
// and the swish gate are applied before the store.
// ---------------------------------------------------------------------------
template <typename Tin, typename To, typename Tg>
__global__ void __launch_bounds__(kThreads)
chunk_out_simt_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k,
                      const Tin* __restrict__ v, SeqLayout L,
                      const int32_t* __restrict__ chunk_base,
                      const float* __restrict__ ws_states, To* __restrict__ out,
                      const Tg* __restrict__ g, const float* __restrict__ gn_w,
                      const float* __restrict__ gn_b, float eps, int gated,
                      int H, int dk, int dv, HeadDecay dec) {
  extern __shared__ float smem[];
  const int ldq = dk + 1;
  float* qs = smem;                        // [kRows][dk+1]
  float* ks = qs + kRows * ldq;            // [kKeys][dk+1]
  float* vs = ks + kKeys * ldq;            // [kKeys][dv]
  float* ss = vs + kKeys * dv;             // [kRows][kKeys+1]
  float* red = ss + kRows * (kKeys + 1);   // [kRows][8] reductions
  __shared__ int row_cs[kRows], row_seq_end[kRows], row_i[kRows];
  __shared__ long long row_slot[kRows];

  const int n0 = blockIdx.x * kRows, h = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  if (tid < kRows) {
    int n = n0 + tid;
    int cs = -1, e = -1, i = 0;
    long long slot = -1;
    if (n < L.Ttot) {
      int s = seq_of_token(L, n);
      int a, b;
      seq_bounds(L, s, a, b);
      if (n >= a && n < b) {
        int c = (n - a) / L.chunk;
        cs = a + c * L.chunk;
        e = b;
        i = n - cs;
        slot = slot_of(L, chunk_base, s, c);
      }
    }
    row_cs[tid] = cs;
    row_seq_end[tid] = e;
    row_i[tid] = i;
    row_slot[tid] = slot;
  }
  for (int e = tid; e < kRows * dk; e += kThreads) {
    int r = e / dk, d = e % dk, n = n0 + r;
    qs[r * ldq + d] = n < L.Ttot ? Io<Tin>::ld(q, (static_cast<size_t>(n) * H + h) * dk + d) : 0.f;
  }
  __syncthreads();

  float acc[kRows];
#pragma unroll
  for (int r = 0; r < kRows; ++r) acc[r] = 0.f;

  // key range shared by the tile: [min chunk start, last row]
  int kbeg = 0x7fffffff, kend = -1;
  for (int r = 0; r < kRows; ++r) {
    if (row_cs[r] >= 0) {
      kbeg = min(kbeg, row_cs[r]);
      kend = max(kend, n0 + r);
    }
  }
  for (int m0 = kbeg; m0 <= kend; m0 += kKeys) {
    __syncthreads();
    for (int e = tid; e < kKeys * dk; e += kThreads) {
      int c = e / dk, d = e % dk, m = m0 + c;
      ks[c * ldq + d] = m <= kend ? Io<Tin>::ld(k, (static_cast<size_t>(m) * H + h) * dk + d) : 0.f;
    }
    for (int e = tid; e < kKeys * dv; e += kThreads) {
      int c = e / dv, d = e % dv, m = m0 + c;
      vs[c * dv + d] = m <= kend ? Io<Tin>::ld(v, (static_cast<size_t>(m) * H + h) * dv + d) : 0.f;
    }
    __syncthreads();
    {
      int r = tid / kKeys, c = tid % kKeys;
      int n = n0 + r, m = m0 + c;
      float sc = 0.f;
      if (row_cs[r] >= 0 && m >= row_cs[r] && m <= n) {
        for (int d = 0; d < dk; ++d) sc = fmaf(qs[r * ldq + d], ks[c * ldq + d], sc);
        sc *= gpow(dec, h, n - m);
      }
      ss[r * (kKeys + 1) + c] = sc;
    }
    __syncthreads();
    if (tid < dv) {
#pragma unroll
      for (int r = 0; r < kRows; ++r) {
        float a = acc[r];
        for (int c = 0; c < kKeys; ++c) a = fmaf(ss[r * (kKeys + 1) + c], vs[c * dv + tid], a);
        acc[r] = a;
      }
    }
  }
  // decayed read of the state entering each row's chunk
  if (tid < dv) {
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      if (row_slot[r] < 0 || row_slot[r] >= L.nslots) continue;
      const float* Sp = ws_states + (static_cast<size_t>(row_slot[r]) * H + h) * dk * dv;
      float a = 0.f;
      for (int d = 0; d < dk; ++d) a = fmaf(qs[r * ldq + d], Sp[static_cast<size_t>(d) * dv + tid], a);
      acc[r] = fmaf(gpow(dec, h, row_i[r] + 1), a, acc[r]);
    }
  }
  if (gated) {
    // per-(row, head) mean, then centred variance, over the dv columns
    float mean[kRows], rstd[kRows];
    for (int pass = 0; pass < 2; ++pass) {
#pragma unroll
      for (int r = 0; r < kRows; ++r) {
        float x = 0.f;
        if (tid < dv) x = pass == 0 ? acc[r] : (acc[r] - mean[r]) * (acc[r] - mean[r]);
        for (int off = 16; off; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
        if (lane == 0) red[r * 8 + warp] = x;
      }
      __syncthreads();
#pragma unroll
      for (int r = 0; r < kRows; ++r) {
        float t = 0.f;
        for (int w = 0; w < 8; ++w) t += red[r * 8 + w];
        if (pass == 0) mean[r] = t / dv;
        else rstd[r] = 1.0f / sqrtf(t / dv + eps);
      }
      __syncthreads();
    }
    if (tid < dv) {
#pragma unroll
      for (int r = 0; r < kRows; ++r) {
        int n = n0 + r;
        if (row_cs[r] < 0) continue;
        size_t idx = (static_cast<size_t>(n) * H + h) * dv + tid;
        float y = (acc[r] - mean[r]) * rstd[r];
        if (gn_w) y *= gn_w[h * dv + tid];
        if (gn_b) y += gn_b[h * dv + tid];
        float gv = Io<Tg>::ld(g, idx);
        y *= gv / (1.0f + expf(-gv));
        Io<To>::st(out, idx, y);
      }
    }
  } else if (tid < dv) {
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      int n = n0 + r;
      if (row_cs[r] < 0) continue;
      Io<To>::st(out, (static_cast<size_t>(n) * H + h) * dv + tid, acc[r]);
    }
  }
}

// ---------------------------------------------------------------------------
// Gradient pass of the backward: block = (16 flat token rows, head h).  Row n
// at position i of its chunk [cs, ce) gets
//   causal (kAnti = false):      out_n = sum_{cs <= m <= n} gamma^(n-m) (a_n.b_m) c_m
//                                        + gamma^(i+1) a_n M
//   anti-causal (kAnti = true):  out_n = sum_{n <= m < ce} gamma^(m-n) (a_n.b_m) c_m
//                                        + gamma^(ce-1-n) a_n M
// where M is the state stored in the workspace slot of the row's chunk: a
// [da][dc] matrix, or with kTrans the transpose of a stored [dc][da] one
// (read through shared memory 32 of its columns at a time, so that the global
// loads stay coalesced).  a, b: [Ttot][H][da]; c, out: [Ttot][H][dc].  Thread
// t owns column t (dc <= 256).
// ---------------------------------------------------------------------------
template <typename Tin, bool kAnti, bool kTrans>
__global__ void __launch_bounds__(kThreads)
chunk_grad_simt_kernel(const Tin* __restrict__ a, const Tin* __restrict__ b,
                       const Tin* __restrict__ c, SeqLayout L,
                       const int32_t* __restrict__ chunk_base,
                       const float* __restrict__ ws_states, float* __restrict__ out, int H,
                       int da, int dc, HeadDecay dec) {
  extern __shared__ float smem[];
  const int lda = da + 1;
  float* as = smem;                        // [kRows][da+1]
  float* bs = as + kRows * lda;            // [kKeys][da+1]
  float* cv = bs + kKeys * lda;            // [kKeys][dc]
  float* ss = cv + kKeys * dc;             // [kRows][kKeys+1]
  float* mt = ss + kRows * (kKeys + 1);    // kTrans: [32][dc+1], 32 columns of M^T
  __shared__ int row_lo[kRows], row_hi[kRows], row_w[kRows];
  __shared__ long long row_slot[kRows];

  const int n0 = blockIdx.x * kRows, h = blockIdx.y;
  const int tid = threadIdx.x;
  if (tid < kRows) {
    // key range [lo, hi] of the row inside its chunk and the exponent of its
    // state weight; lo > hi marks a row outside every sequence
    const int n = n0 + tid;
    int lo = 1, hi = 0, w = 0;
    long long slot = -1;
    if (n < L.Ttot) {
      const int sq = seq_of_token(L, n);
      int sa, sb;
      seq_bounds(L, sq, sa, sb);
      if (n >= sa && n < sb) {
        const int ch = (n - sa) / L.chunk;
        const int cs = sa + ch * L.chunk;
        const int ce = min(cs + L.chunk, sb);
        if (kAnti) {
          lo = n; hi = ce - 1; w = ce - 1 - n;
        } else {
          lo = cs; hi = n; w = n - cs + 1;
        }
        slot = slot_of(L, chunk_base, sq, ch);
      }
    }
    row_lo[tid] = lo;
    row_hi[tid] = hi;
    row_w[tid] = w;
    row_slot[tid] = slot;
  }
  for (int e = tid; e < kRows * da; e += kThreads) {
    const int r = e / da, d = e % da, n = n0 + r;
    as[r * lda + d] = n < L.Ttot ? Io<Tin>::ld(a, (static_cast<size_t>(n) * H + h) * da + d) : 0.f;
  }
  __syncthreads();

  float acc[kRows];
#pragma unroll
  for (int r = 0; r < kRows; ++r) acc[r] = 0.f;
  int kbeg = 0x7fffffff, kend = -1;
  for (int r = 0; r < kRows; ++r) {
    if (row_lo[r] <= row_hi[r]) {
      kbeg = min(kbeg, row_lo[r]);
      kend = max(kend, row_hi[r]);
    }
  }
  for (int m0 = kbeg; m0 <= kend; m0 += kKeys) {
    __syncthreads();
    for (int e = tid; e < kKeys * da; e += kThreads) {
      const int j = e / da, d = e % da, m = m0 + j;
      bs[j * lda + d] = m <= kend ? Io<Tin>::ld(b, (static_cast<size_t>(m) * H + h) * da + d) : 0.f;
    }
    for (int e = tid; e < kKeys * dc; e += kThreads) {
      const int j = e / dc, d = e % dc, m = m0 + j;
      cv[j * dc + d] = m <= kend ? Io<Tin>::ld(c, (static_cast<size_t>(m) * H + h) * dc + d) : 0.f;
    }
    __syncthreads();
    {
      const int r = tid / kKeys, j = tid % kKeys;
      const int n = n0 + r, m = m0 + j;
      float sc = 0.f;
      if (m >= row_lo[r] && m <= row_hi[r]) {
        for (int d = 0; d < da; ++d) sc = fmaf(as[r * lda + d], bs[j * lda + d], sc);
        sc *= gpow(dec, h, kAnti ? m - n : n - m);
      }
      ss[r * (kKeys + 1) + j] = sc;
    }
    __syncthreads();
    if (tid < dc) {
#pragma unroll
      for (int r = 0; r < kRows; ++r) {
        float x = acc[r];
        for (int j = 0; j < kKeys; ++j) x = fmaf(ss[r * (kKeys + 1) + j], cv[j * dc + tid], x);
        acc[r] = x;
      }
    }
  }
  // decayed read of the state of each row's chunk
  if (kTrans) {
    // rows of the block share at most a few slots: walk the distinct ones
    float t[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r) t[r] = 0.f;
    for (int r0 = 0; r0 < kRows; ++r0) {
      const long long slot = row_slot[r0];
      bool first = row_lo[r0] <= row_hi[r0] && slot >= 0 && slot < L.nslots;
      for (int r = 0; r < r0 && first; ++r)
        if (row_slot[r] == slot && row_lo[r] <= row_hi[r]) first = false;
      if (!first) continue;                      // uniform over the block
      const float* M = ws_states + (static_cast<size_t>(slot) * H + h) * da * dc;
      for (int d0 = 0; d0 < da; d0 += 32) {
        __syncthreads();
        for (int e = tid; e < 32 * dc; e += kThreads) {
          const int tt = e >> 5, j = e & 31;       // 32 consecutive d of column tt
          mt[j * (dc + 1) + tt] = d0 + j < da ? M[static_cast<size_t>(tt) * da + d0 + j] : 0.f;
        }
        __syncthreads();
        if (tid < dc) {
#pragma unroll
          for (int r = 0; r < kRows; ++r) {
            if (row_slot[r] != slot) continue;
            float x = t[r];
            const int jn = min(32, da - d0);
            for (int j = 0; j < jn; ++j) x = fmaf(as[r * lda + d0 + j], mt[j * (dc + 1) + tid], x);
            t[r] = x;
          }
        }
      }
    }
    if (tid < dc) {
#pragma unroll
      for (int r = 0; r < kRows; ++r) {
        if (row_lo[r] > row_hi[r]) continue;
        float x = acc[r];
        if (row_slot[r] >= 0 && row_slot[r] < L.nslots) x = fmaf(gpow(dec, h, row_w[r]), t[r], x);
        out[(static_cast<size_t>(n0 + r) * H + h) * dc + tid] = x;
      }
    }
    return;
  }
  if (tid < dc) {
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      const int n = n0 + r;
      if (row_lo[r] > row_hi[r]) continue;
      float x = acc[r];
      if (row_slot[r] >= 0 && row_slot[r] < L.nslots) {
        const float* M = ws_states + (static_cast<size_t>(row_slot[r]) * H + h) * da * dc;
        float t = 0.f;
        for (int d = 0; d < da; ++d) t = fmaf(as[r * lda + d], M[static_cast<size_t>(d) * dc + tid], t);
        x = fmaf(gpow(dec, h, row_w[r]), t, x);
      }
      out[(static_cast<size_t>(n) * H + h) * dc + tid] = x;
    }
  }
}

template <typename Tin>
cudaError_t launch_state_pass(bool rev, const void* k, const void* v, const SeqLayout& L,
                              const int32_t* chunk_base, const float* state_in, float* state_out,
                              float* states, int H, int dk, int dv, const HeadDecay& dec,
                              cudaStream_t s) {
  const size_t smem = sizeof(float) * (kStateTok * dk + kStateTok * 32);
  auto kern = rev ? chunk_state_simt_kernel<Tin, true> : chunk_state_simt_kernel<Tin, false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid((dv + 31) / 32, H, L.nseq);
  kern<<<grid, kThreads, smem, s>>>(static_cast<const Tin*>(k), static_cast<const Tin*>(v), L,
                                    chunk_base, state_in, state_out, states, H, dk, dv, dec);
  return cudaGetLastError();
}

template <typename Tin, bool kAnti, bool kTrans>
cudaError_t launch_grad_pass(const void* a, const void* b, const void* c, const SeqLayout& L,
                             const int32_t* chunk_base, const float* states, float* out, int H,
                             int da, int dc, const HeadDecay& dec, cudaStream_t s) {
  const size_t smem =
      sizeof(float) * ((kRows + kKeys) * (da + 1) + kKeys * dc + kRows * (kKeys + 1) +
                       (kTrans ? 32 * (dc + 1) : 0));
  auto kern = chunk_grad_simt_kernel<Tin, kAnti, kTrans>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid((L.Ttot + kRows - 1) / kRows, H);
  kern<<<grid, kThreads, smem, s>>>(static_cast<const Tin*>(a), static_cast<const Tin*>(b),
                                    static_cast<const Tin*>(c), L, chunk_base, states, out, H, da,
                                    dc, dec);
  return cudaGetLastError();
}

// The backward in five launches: the forward states S (entering each chunk),
// the states of the future F (after each chunk, walked backwards, ending in
// d_state_in), then dQ (causal, reads S^T), dV (anti-causal, reads F) and dK
// (anti-causal, reads F^T).
template <typename Tin>
cudaError_t chunkwise_bwd_typed(const void* q, const void* k, const void* v, const void* d_out,
                                const SeqLayout& L, const float* state_in,
                                const float* d_state_out, float* dq, float* dk, float* dv,
                                float* d_state_in, const ChunkBwdWorkspace& ws, int H, int dk_,
                                int dv_, const HeadDecay& dec, cudaStream_t s) {
  cudaError_t e = launch_state_pass<Tin>(false, k, v, L, ws.chunk_base, state_in, nullptr,
                                         ws.fwd_states, H, dk_, dv_, dec, s);
  if (e == cudaSuccess)
    e = launch_state_pass<Tin>(true, q, d_out, L, ws.chunk_base, d_state_out, d_state_in,
                               ws.bwd_states, H, dk_, dv_, dec, s);
  if (e != cudaSuccess || L.Ttot == 0) return e;
  e = launch_grad_pass<Tin, false, true>(d_out, v, k, L, ws.chunk_base, ws.fwd_states, dq, H,
                                         dv_, dk_, dec, s);
  if (e == cudaSuccess)
    e = launch_grad_pass<Tin, true, false>(k, q, d_out, L, ws.chunk_base, ws.bwd_states, dv, H,
                                           dk_, dv_, dec, s);
  if (e == cudaSuccess)
    e = launch_grad_pass<Tin, true, true>(v, d_out, q, L, ws.chunk_base, ws.bwd_states, dk, H,
                                          dv_, dk_, dec, s);
  return e;
}

template <typename Tin, typename To>
cudaError_t parallel_typed(const void* q, const void* k, const void* v, void* o, int B, int T,
                           int H, int dk, int dv, const HeadDecay& dec, cudaStream_t s) {
  size_t smem = sizeof(float) * (2 * kRows * (dk + 1) + kKeys * dv + kRows * (kKeys + 1));
  auto kern = parallel_simt_kernel<Tin, To>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid((T + kRows - 1) / kRows, H, B);
  kern<<<grid, kThreads, smem, s>>>(static_cast<const Tin*>(q), static_cast<const Tin*>(k),
                                    static_cast<const Tin*>(v), static_cast<To*>(o), T, H, dk,
                                    dv, dec);
  return cudaGetLastError();
}

template <typename Tin, typename To, typename Tg>
cudaError_t chunkwise_typed(int phases, const void* q, const void* k, const void* v,
                            const SeqLayout& L,
                            const float* state_in, float* state_out, void* out, const void* g,
                            const float* gn_w, const float* gn_b, float eps, bool gated,
                            ChunkWorkspace ws, int H, int dk, int dv, const HeadDecay& dec,
                            cudaStream_t s) {
  if (phases & 1) {
    size_t smem = sizeof(float) * (kStateTok * dk + kStateTok * 32);
    auto kern = chunk_state_simt_kernel<Tin, false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    dim3 grid((dv + 31) / 32, H, L.nseq);
    kern<<<grid, kThreads, smem, s>>>(static_cast<const Tin*>(k), static_cast<const Tin*>(v), L,
                                      ws.chunk_base, state_in, state_out,
                                      static_cast<float*>(ws.states), H, dk, dv, dec);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (L.Ttot == 0 || !(phases & 2)) return cudaSuccess;
  size_t smem = sizeof(float) * (2 * kRows * (dk + 1) + kKeys * dv + kRows * (kKeys + 1) +
                                 kRows * 8);
  auto kern = chunk_out_simt_kernel<Tin, To, Tg>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid((L.Ttot + kRows - 1) / kRows, H);
  kern<<<grid, kThreads, smem, s>>>(static_cast<const Tin*>(q), static_cast<const Tin*>(k),
                                    static_cast<const Tin*>(v), L, ws.chunk_base,
                                    static_cast<const float*>(ws.states), static_cast<To*>(out),
                                    static_cast<const Tg*>(g), gn_w, gn_b, eps, gated ? 1 : 0,
                                    H, dk, dv, dec);
  return cudaGetLastError();
}

}  // namespace

size_t chunkwise_meta_bytes(int nseq) {
  // chunk_base [nseq+1] | longest-first sequence order [nseq]
  size_t b = sizeof(int32_t) * (2 * static_cast<size_t>(nseq) + 1);
  return (b + 255) / 256 * 256;
}

cudaError_t launch_parallel_simt(const void* q, const void* k, const void* v, DType in_t,
                                 void* o, DType o_t, int B, int T, int H, int dk, int dv,
                                 const HeadDecay& dec, cudaStream_t s) {
  using bf = __nv_bfloat16;
  if (in_t == DType::F32)
    return o_t == DType::F32 ? parallel_typed<float, float>(q, k, v, o, B, T, H, dk, dv, dec, s)
                             : parallel_typed<float, bf>(q, k, v, o, B, T, H, dk, dv, dec, s);
  return o_t == DType::F32 ? parallel_typed<bf, float>(q, k, v, o, B, T, H, dk, dv, dec, s)
                           : parallel_typed<bf, bf>(q, k, v, o, B, T, H, dk, dv, dec, s);
}

cudaError_t launch_chunk_prep(const SeqLayout& L, ChunkWorkspace ws, unsigned* err,
                              cudaStream_t s) {
  if (L.cu == nullptr) return cudaSuccess;
  chunk_prep_kernel<<<1, 1024, 0, s>>>(L, ws.chunk_base, ws.order, err);
  return cudaGetLastError();
}

cudaError_t launch_chunkwise_simt(int phases, const void* q, const void* k, const void* v,
                                  DType in_t,
                                  const SeqLayout& L, const float* state_in, float* state_out,
                                  void* out, DType out_t, const void* g, DType g_t,
                                  const float* gn_w, const float* gn_b, float eps, bool gated,
                                  ChunkWorkspace ws, int H, int dk, int dv,
                                  const HeadDecay& dec, unsigned* err, cudaStream_t s) {
  (void)err;
  if (in_t != DType::F32) return cudaErrorInvalidValue;
  using bf = __nv_bfloat16;
  if (out_t == DType::F32)
    return g_t == DType::F32
               ? chunkwise_typed<float, float, float>(phases, q, k, v, L, state_in, state_out, out, g,
                                                      gn_w, gn_b, eps, gated, ws, H, dk, dv,
                                                      dec, s)
               : chunkwise_typed<float, float, bf>(phases, q, k, v, L, state_in, state_out, out, g,
                                                   gn_w, gn_b, eps, gated, ws, H, dk, dv, dec,
                                                   s);
  return g_t == DType::F32
             ? chunkwise_typed<float, bf, float>(phases, q, k, v, L, state_in, state_out, out, g, gn_w,
                                                 gn_b, eps, gated, ws, H, dk, dv, dec, s)
             : chunkwise_typed<float, bf, bf>(phases, q, k, v, L, state_in, state_out, out, g, gn_w,
                                              gn_b, eps, gated, ws, H, dk, dv, dec, s);
}

cudaError_t launch_chunkwise_bwd_simt(const void* q, const void* k, const void* v,
                                      const void* d_out, DType in_t, const SeqLayout& L,
                                      const float* state_in, const float* d_state_out, float* dq,
                                      float* dk, float* dv, float* d_state_in,
                                      const ChunkBwdWorkspace& ws, int H, int dk_, int dv_,
                                      const HeadDecay& dec, cudaStream_t s) {
  if (in_t == DType::F32)
    return chunkwise_bwd_typed<float>(q, k, v, d_out, L, state_in, d_state_out, dq, dk, dv,
                                      d_state_in, ws, H, dk_, dv_, dec, s);
  return chunkwise_bwd_typed<__nv_bfloat16>(q, k, v, d_out, L, state_in, d_state_out, dq, dk, dv,
                                            d_state_in, ws, H, dk_, dv_, dec, s);
}

}  // namespace ret

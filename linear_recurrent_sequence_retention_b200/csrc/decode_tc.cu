// Several recurrent decode steps per pass over the state, on the tensor cores
// (bf16 q, k, v; float32 state).  The recurrence of the abeam.tech summary of
// Sun et al. 2023 (section 「学習は並列、生成は状態更新」), unrolled over Tn
// tokens entering with state S (the same form as decode.cu):
//     o_t = gamma^(t+1) q_t S + sum_{j<=t} gamma^(t-j) (q_t . k_j) v_j
//     S'  = gamma^Tn S + sum_j gamma^(Tn-1-j) k_j^T v_j
// Both products that touch every state element are matrix products with Tn
// (<= 16) on the short side: O^T = S^T Q^T (M = 128 columns of d_v per block,
// K = d_k, N = 16 tokens) and dS = (zeta K)^T V (M = 128 rows of d_k, K = 16
// tokens, N = 128 columns), so both run as tcgen05 MMAs of kind::tf32 on
// float32 operands in shared memory; S' = gamma^Tn S + dS is formed in float32
// by CUDA cores and leaves through TMA.  The state itself stays float32 (only
// the MMA operands are read at tf32 precision, relative error 2^-11), which
// keeps the outputs and the carried state well inside the bf16-input bound.
//
// Persistent: one CTA per SM walks the (n, h) states.  Warp 0 streams, through
// a ring of 32 KB stages, first the item's q, k, v rows (bf16, one stage, TMA)
// and then its state (64 rows x 128 columns per stage, TMA, 128-byte swizzle
// with 32-byte atoms, the layout MN-major tf32 operands take); warp 1 issues
// the MMAs; warps 2..9 form q_t gamma^(t+1), zeta_j k_j and v as float32
// operand tiles from the q, k, v stage (and the Tn x Tn intra-step scores, by
// mma.sync on four warps), update every state stage in place after its read
// MMA, store it back with TMA and finally add the intra-step terms to the
// outputs.  Every wait is bounded.
#include <cudaTypedefs.h>

#include "launch.h"
#include "tc_ptx.cuh"

namespace ret {
namespace {

using namespace tc;

constexpr int kDtThreads = 320;                 // warp 0 TMA, warp 1 MMA, warps 2..9 workers
constexpr int kDtStages = 5;
constexpr uint32_t kDtBox = 8192;               // [64 state rows][32 float32]
constexpr uint32_t kDtStage = 4 * kDtBox;       // 64 state rows x 128 columns
constexpr uint32_t kDtChunk = 2048;             // [16 token rows][32 float32]
constexpr int kDtMaxT = 16;

struct DecTcParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  void* o;
  int o_bf16;
  int nitems, Tn, H, dk, dv;
  HeadDecay dec;
  unsigned* err;
};

struct DtLayout {
  uint32_t qs, zk, vb, att, bars, smem;
  __host__ __device__ DtLayout(int dk, int dv) {
    qs = kDtStages * kDtStage;                          // [dk/32 chunks][16 rows][128 B]
    zk = qs + (dk / 32) * kDtChunk;                     // same shape
    vb = zk + (dk / 32) * kDtChunk;                     // [dv/32 chunks][16 rows][128 B]
    att = vb + (dv / 32) * kDtChunk;                    // [16][16] float, then [2][16] decay factors
    bars = att + kDtMaxT * kDtMaxT * 4 + 2 * kDtMaxT * 4;
    smem = bars + 256;
  }
};

// Byte offset of element (row, col) in a tile of 32-float (128-byte) rows with
// the 128-byte swizzle of 16-byte atoms (K-major tf32 operands): the 16-byte
// piece index is XORed with row mod 8.
__device__ __forceinline__ uint32_t sw_off(int row, int col) {
  return static_cast<uint32_t>(row * 128 + ((((col & 31) >> 2) ^ (row & 7)) << 4) + (col & 3) * 4);
}
// The same with 32-byte atoms (MN-major tf32 operands, and the TMA mode
// "128-byte swizzle, 32-byte atoms"): the 32-byte piece index is XORed with
// row mod 4.
__device__ __forceinline__ uint32_t sw32_off(int row, int col) {
  return static_cast<uint32_t>(row * 128 + ((((col & 31) >> 3) ^ (row & 3)) << 5) + (col & 7) * 4);
}
// Shared-memory descriptor of an MN-major tf32 operand in that layout (layout
// type 1): LBO = distance between 32-element M/N chunks, SBO = distance between
// 4-row K groups.
__device__ __forceinline__ uint64_t sdesc_sw128_atom32(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= 1ull << 46;
  d |= 1ull << 61;
  return d;
}

__device__ __forceinline__ bool wall(bool v) { return __all_sync(0xffffffffu, v) != 0; }

__global__ void __launch_bounds__(kDtThreads, 1)
decode_multi_tc_kernel(const __grid_constant__ CUtensorMap tmS, const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                       const DecTcParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const DtLayout lay(p.dk, p.dv);
  uint8_t* ring = smem;
  uint8_t* qs = smem + lay.qs;
  uint8_t* zk = smem + lay.zk;
  uint8_t* vb = smem + lay.vb;
  float* att = reinterpret_cast<float*>(smem + lay.att);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + lay.bars);
  uint64_t* empty = full + kDtStages;       // the stage's update has been stored
  uint64_t* mma_done = empty + kDtStages;   // the read MMA of the stage is complete
  uint64_t* du_full = mma_done + kDtStages; // [2] dS of an M-block is in TMEM
  uint64_t* du_free = du_full + 2;          // [2] the workers have read it
  uint64_t* pro_full = du_free + 2;         // the item's operand tiles are formed
  uint64_t* do_full = pro_full + 1;         // every MMA of the item is complete
  uint64_t* do_free = do_full + 1;          // the item's outputs have been read from TMEM
  uint64_t* drain = do_free + 1;
  uint32_t* tmem_hold = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_hold + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nb = p.dv / 128, nm = p.dk / 128, nq = p.dk / 64;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kDtStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
      mbar_init(&mma_done[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&du_full[i], 1);
      mbar_init(&du_free[i], 8);
    }
    mbar_init(pro_full, 8);
    mbar_init(do_full, 1);
    mbar_init(do_free, 8);
    mbar_init(drain, 1);
    *abort_flag = 0;
    if ((smem_u32(smem) & 1023u) != 0) {
      *abort_flag = 1;
      raise_error(p.err, kErrTimeout);
    }
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_hold, 512);    // dS in columns [0, 256) (two buffers), O^T blocks from 256
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_hold;

  if (warp == 0) {
    // ---------------- TMA producer: per item the q, k, v stage, then the state ----------------
    // (64 rows x 128 columns per stage)
    if (lane == 0 && !*abort_flag) {
      tma_prefetch_desc(&tmS);
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int it = 0;
      bool ok = true;
      const uint32_t qkv_bytes = static_cast<uint32_t>(p.Tn * (2 * p.dk + p.dv) * 2);
      for (int item = blockIdx.x; item < p.nitems && ok; item += gridDim.x) {
        {
          // the item's q, k and v rows (bf16, [Tn][dk], [Tn][dk], [dv/128][Tn][128]) into one stage
          const int st = it % kDtStages;
          if (!mbar_wait(&empty[st], ((it / kDtStages) & 1) ^ 1, abort_flag, p.err)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[st], qkv_bytes);
          uint8_t* dst = ring + st * kDtStage;
          const int h = item % p.H, y0 = (item / p.H) * p.Tn;
          tma_load_2d(dst, &tmQ, &full[st], h * p.dk, y0);
          tma_load_2d(dst + p.Tn * p.dk * 2, &tmK, &full[st], h * p.dk, y0);
          for (int vbx = 0; vbx < p.dv / 128; ++vbx)
            tma_load_2d(dst + 2 * p.Tn * p.dk * 2 + vbx * p.Tn * 256, &tmV, &full[st], h * p.dv + 128 * vbx, y0);
          ++it;
        }
        // row-block major: the d_v blocks of the same 128 state rows go out one
        // after another, so the four 512-byte pieces of each 2 KB state row are
        // fetched two stages apart (four in column-block order)
        for (int mb = 0; mb < nm && ok; ++mb)
        for (int b = 0; b < nb && ok; ++b) {
          for (int q2 = 0; q2 < 2; ++q2, ++it) {
            const int q = 2 * mb + q2;
            const int st = it % kDtStages;
            if (!mbar_wait(&empty[st], ((it / kDtStages) & 1) ^ 1, abort_flag, p.err)) { ok = false; break; }
            mbar_arrive_expect_tx(&full[st], kDtStage);
            for (int c = 0; c < 4; ++c)
              tma_load_2d(ring + st * kDtStage + c * kDtBox, &tmS, &full[st], 128 * b + 32 * c,
                          item * p.dk + 64 * q);
          }
        }
      }
      if (!ok) {
        for (int j = 1; j <= kDtStages && it - j >= 0; ++j) {
          const int i2 = it - j;
          mbar_wait_drain(&full[i2 % kDtStages], (i2 / kDtStages) & 1);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0 && !*abort_flag) {
      constexpr uint32_t id_upd = idesc_tf32_f32(128, 128, true, true);
      constexpr uint32_t id_rd = idesc_tf32_f32(128, 16, true, false);
      const uint32_t ring_a = smem_u32(ring), qs_a = smem_u32(qs), zk_a = smem_u32(zk),
                     vb_a = smem_u32(vb);
      int it = 0, ndu = 0, nitem = 0;
      bool ok = true, issued = false;
      for (int item = blockIdx.x; item < p.nitems && ok; item += gridDim.x, ++nitem) {
        ++it;                                   // the item's q, k, v stage (the workers' own)
        if (!mbar_wait(pro_full, nitem & 1, abort_flag, p.err)) { ok = false; break; }
        if (nitem > 0 && !mbar_wait(do_free, (nitem - 1) & 1, abort_flag, p.err)) { ok = false; break; }
        tc_fence_after();
        for (int mb = 0; mb < nm && ok; ++mb) {
          for (int b = 0; b < nb && ok; ++b, ++ndu) {
            const int u = ndu & 1;
            if (ndu >= 2 && !mbar_wait(&du_free[u], ((ndu >> 1) + 1) & 1, abort_flag, p.err)) { ok = false; break; }
            tc_fence_after();
            // dS rows 128mb.., columns 128b..: (zeta K)^T [128 x 16] V [16 x 128]
#pragma unroll
            for (int ks = 0; ks < 2; ++ks)
              mma_tf32(tmem + 128 * u,
                       sdesc_sw128_atom32(zk_a + 4 * mb * kDtChunk + ks * 1024, kDtChunk, 512),
                       sdesc_sw128_atom32(vb_a + 4 * b * kDtChunk + ks * 1024, kDtChunk, 512), id_upd,
                       ks > 0);
            issued = true;
            mma_commit(&du_full[u]);
            for (int q2 = 0; q2 < 2; ++q2, ++it) {
              const int q = 2 * mb + q2;
              const int st = it % kDtStages;
              if (!mbar_wait(&full[st], (it / kDtStages) & 1, abort_flag, p.err)) { ok = false; break; }
              tc_fence_after();
              // O^T[block b] += S^T (128 columns x 64 rows of d_k) Q^T (64 rows x 16 tokens)
              const uint32_t sa = ring_a + st * kDtStage;
#pragma unroll
              for (int ks = 0; ks < 8; ++ks) {
                const int kg = 64 * q + 8 * ks;
                mma_tf32(tmem + 256 + 16 * b, sdesc_sw128_atom32(sa + ks * 1024, kDtBox, 512),
                         sdesc_sw128(qs_a + (kg >> 5) * kDtChunk + (kg & 31) * 4, 16, 1024), id_rd,
                         q > 0 || ks > 0);
              }
              mma_commit(&mma_done[st]);
            }
          }
        }
        if (!ok) break;
        mma_commit(do_full);
      }
      if (!ok && issued) {
        mma_commit(drain);
        mbar_wait_drain(drain, 0);
      }
    }
  } else {
    // ---------------- workers: warps 2..9 ----------------
    const int w = warp - 2;                 // 0..7
    const int quad = warp & 3;              // TMEM lane quadrant of this warp
    const int half = w >> 2;                // column half of a stage / block parity of the outputs
    const int set = (quad >> 1);            // stages with q2 == set (TMEM lanes 64 set ..)
    const int rr = 32 * (quad & 1) + lane;  // row within a stage
    const int wt = threadIdx.x - 64;        // 0..255
    const bool store_leader = quad == 2 * set && half == 0 && lane == 0;
    int it = 0, ndu = 0, nitem = 0;
    int pend_st = -1;      // (store leader) the item's last stage, released after the outputs
    bool ok = true;
    for (int item = blockIdx.x; item < p.nitems; item += gridDim.x, ++nitem) {
      // uniform over the 256 workers: the named barriers below stay matched
      uint32_t r;
      asm volatile(
          "{\n\t.reg .pred a, b;\n\t"
          "setp.ne.u32 a, %1, 0;\n\t"
          "bar.red.and.pred b, 1, 256, a;\n\t"
          "selp.u32 %0, 1, 0, b;\n\t}"
          : "=r"(r)
          : "r"((ok && !*abort_flag) ? 1u : 0u)
          : "memory");
      if (!r) break;
      const int h = item % p.H, n = item / p.H;
      const Decay1 dg(p.dec, h);
      const int qkv_it = it++;
      const uint8_t* qkv = ring + (qkv_it % kDtStages) * kDtStage;
      const bool qkv_ok = wall(ok && mbar_wait(&full[qkv_it % kDtStages], (qkv_it / kDtStages) & 1, abort_flag, p.err));
      if (!qkv_ok) ok = false;
      // (a) q and k of the Tn tokens, unscaled, as [16][dk] float32 rows in the
      // qs and zk regions (k's float4 columns XOR-swizzled by row, so that the
      // score pass below reads 16 rows without bank conflicts; zero rows from Tn
      // on); v straight into its MN-major tile; the per-token decay factors.
      // The rows come from the item's q, k, v ring stage; every 16-byte load
      // is issued before the first store.
      float* qraw = reinterpret_cast<float*>(qs);
      float* kraw = reinterpret_cast<float*>(zk);
      float* fac = att + kDtMaxT * kDtMaxT;            // [2][16]: gamma^(t+1), zeta_t
      auto cvt8 = [](uint4 u, float (&x)[8]) {
        const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          x[2 * e] = __uint_as_float(w4[e] << 16);
          x[2 * e + 1] = __uint_as_float(w4[e] & 0xffff0000u);
        }
      };
      {
        constexpr int kQK = kDtMaxT * 256 / 8 / 256;     // 16-byte vectors of q (and of k) per thread at d_k = 256
        constexpr int kV = kDtMaxT * 512 / 8 / 256;      // of v at d_v = 512
        const int nv = kDtMaxT * p.dv / 8;
        uint4 uq[kQK], uk[kQK], uv[kV];
#pragma unroll
        for (int m = 0; m < kQK; ++m) {
          const int e8 = (wt + 256 * m) * 8, t = e8 / p.dk, i = e8 % p.dk;
          uq[m] = uk[m] = make_uint4(0, 0, 0, 0);
          if (e8 < kDtMaxT * p.dk && t < p.Tn && qkv_ok) {
            uq[m] = *reinterpret_cast<const uint4*>(qkv + (t * p.dk + i) * 2);
            uk[m] = *reinterpret_cast<const uint4*>(qkv + ((p.Tn + t) * p.dk + i) * 2);
          }
        }
        for (int m0 = 0; m0 < nv; m0 += kV * 256) {
#pragma unroll
          for (int m = 0; m < kV; ++m) {
            const int e8 = (m0 + wt + 256 * m) * 8, t = e8 / p.dv, cc = e8 % p.dv;
            uv[m] = make_uint4(0, 0, 0, 0);
            if (e8 < kDtMaxT * p.dv && t < p.Tn && qkv_ok)
              uv[m] = *reinterpret_cast<const uint4*>(qkv + 2 * p.Tn * p.dk * 2 + (cc >> 7) * p.Tn * 256 +
                                                      (t * 128 + (cc & 127)) * 2);
          }
#pragma unroll
          for (int m = 0; m < kV; ++m) {
            const int e8 = (m0 + wt + 256 * m) * 8, t = e8 / p.dv, cc = e8 % p.dv;
            if (e8 >= kDtMaxT * p.dv) continue;
            float xv[8];
            cvt8(uv[m], xv);
            // 8 consecutive columns (cc mod 8 == 0) are one 32-byte atom
            float4* dv4 = reinterpret_cast<float4*>(vb + (cc >> 5) * kDtChunk + sw32_off(t, cc));
            dv4[0] = make_float4(xv[0], xv[1], xv[2], xv[3]);
            dv4[1] = make_float4(xv[4], xv[5], xv[6], xv[7]);
          }
        }
#pragma unroll
        for (int m = 0; m < kQK; ++m) {
          const int e8 = (wt + 256 * m) * 8, t = e8 / p.dk, i = e8 % p.dk;
          if (e8 >= kDtMaxT * p.dk) continue;
          float xq[8], xk[8];
          cvt8(uq[m], xq);
          cvt8(uk[m], xk);
          float4* dq = reinterpret_cast<float4*>(qraw + t * p.dk + i);
          dq[0] = make_float4(xq[0], xq[1], xq[2], xq[3]);
          dq[1] = make_float4(xq[4], xq[5], xq[6], xq[7]);
          float4* kr = reinterpret_cast<float4*>(kraw + t * p.dk);
          const int c4 = i >> 2;                       // float4 column, swizzled by row t
          kr[c4 ^ (t & 7)] = make_float4(xk[0], xk[1], xk[2], xk[3]);
          kr[(c4 + 1) ^ (t & 7)] = make_float4(xk[4], xk[5], xk[6], xk[7]);
        }
        if (wt < kDtMaxT) {
          fac[wt] = wt < p.Tn ? dg.pow(wt + 1) : 0.f;
          fac[kDtMaxT + wt] = wt < p.Tn ? dg.pow(p.Tn - 1 - wt) : 0.f;
        }
      }
      asm volatile("bar.sync 2, 256;" ::: "memory");
      if (wt == 0) {                                   // the q, k, v stage is read
        mbar_arrive(&empty[qkv_it % kDtStages]);
        mbar_arrive(&mma_done[qkv_it % kDtStages]);    // keeps that barrier's phases in step with the ring
      }
      // (b) intra-step scores (q_t . k_j) gamma^(t-j), j <= t, on the tensor
      // cores (mma.sync m16n8k8, tf32: q and k are bf16 values, exact in tf32):
      // warp w < 4 forms the 16 x 8 tile of keys 8 (w & 1).. over half of d_k
      // (w >> 1); the second half's tile passes through att
      if (w < 4) {
        const int nt = w & 1, kh = w >> 1;
        const int g = lane >> 2, tq = lane & 3;
        const int jrow = 8 * nt + g;                    // key of this thread's B values
        const float* qa = qraw + g * p.dk;
        const float* qb = qraw + (g + 8) * p.dk;
        const float* kr = kraw + jrow * p.dk;
        float c[4] = {0.f, 0.f, 0.f, 0.f};
        const int kbeg = kh * (p.dk / 2), kend = kbeg + p.dk / 2;
        for (int k0 = kbeg; k0 < kend; k0 += 8) {
          const int c0 = k0 + tq, c1 = k0 + tq + 4;
          const uint32_t a0 = __float_as_uint(qa[c0]), a1 = __float_as_uint(qb[c0]);
          const uint32_t a2 = __float_as_uint(qa[c1]), a3 = __float_as_uint(qb[c1]);
          const uint32_t b0 = __float_as_uint(kr[(((c0 >> 2) ^ (jrow & 7)) << 2) + (c0 & 3)]);
          const uint32_t b1 = __float_as_uint(kr[(((c1 >> 2) ^ (jrow & 7)) << 2) + (c1 & 3)]);
          asm volatile(
              "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, "
              "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
              : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
              : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
        }
        const int j0 = 8 * nt + 2 * tq;
        if (kh == 1) {
          att[g * kDtMaxT + j0] = c[0];
          att[g * kDtMaxT + j0 + 1] = c[1];
          att[(g + 8) * kDtMaxT + j0] = c[2];
          att[(g + 8) * kDtMaxT + j0 + 1] = c[3];
        }
        asm volatile("bar.sync 5, 128;" ::: "memory");
        if (kh == 0) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int t = g + 8 * (e >> 1), j = j0 + (e & 1);
            const float x = c[e] + att[t * kDtMaxT + j];
            att[t * kDtMaxT + j] = (j <= t && t < p.Tn) ? x * dg.pow(t - j) : 0.f;
          }
        }
      }
      // (c) the same elements rewritten in place as the MMA operand tiles:
      // q_t gamma^(t+1) (K-major, 16-byte atoms) and zeta_t k_t (MN-major,
      // 32-byte atoms), four consecutive elements at a time; every thread reads
      // its elements before any writes
      {
        constexpr int kF4 = kDtMaxT * 256 / 4 / 256;     // float4 per thread at d_k = 256
        float4 qv[kF4], kv[kF4];
#pragma unroll
        for (int m = 0; m < kF4; ++m) {
          const int e4 = (wt + 256 * m) * 4, t = e4 / p.dk, i = e4 % p.dk;
          if (e4 < kDtMaxT * p.dk) {
            qv[m] = *reinterpret_cast<const float4*>(qraw + e4);
            kv[m] = reinterpret_cast<const float4*>(kraw + t * p.dk)[(i >> 2) ^ (t & 7)];
          }
        }
        asm volatile("bar.sync 2, 256;" ::: "memory");
#pragma unroll
        for (int m = 0; m < kF4; ++m) {
          const int e4 = (wt + 256 * m) * 4, t = e4 / p.dk, i = e4 % p.dk;
          if (e4 >= kDtMaxT * p.dk) continue;
          const float sq = fac[t], sk = fac[kDtMaxT + t];
          float4 a = qv[m], c = kv[m];
          a.x *= sq; a.y *= sq; a.z *= sq; a.w *= sq;
          c.x *= sk; c.y *= sk; c.z *= sk; c.w *= sk;
          *reinterpret_cast<float4*>(qs + (i >> 5) * kDtChunk + sw_off(t, i)) = a;
          *reinterpret_cast<float4*>(zk + (i >> 5) * kDtChunk + sw32_off(t, i)) = c;
        }
      }
      fence_proxy_async_smem();
      asm volatile("bar.sync 2, 256;" ::: "memory");
      if (lane == 0) mbar_arrive(pro_full);

      // stages: S' = gamma^Tn S + dS in place, then back to global memory
      const float gT = dg.pow(p.Tn);
      for (int mb = 0; mb < nm; ++mb) {
        for (int b = 0; b < nb; ++b, ++ndu) {
          const int u = ndu & 1;
          for (int q2 = 0; q2 < 2; ++q2, ++it) {
            const int q = 2 * mb + q2;
            const int st = it % kDtStages;
            if (q2 != set) continue;
            uint8_t* stg = ring + st * kDtStage;
            bool go = ok;
            go = wall(go && mbar_wait(&du_full[u], (ndu >> 1) & 1, abort_flag, p.err));
            go = wall(go && mbar_wait(&mma_done[st], (it / kDtStages) & 1, abort_flag, p.err));
            if (go) {
              tc_fence_after();
              for (int cc = 0; cc < 2; ++cc) {
                const int c = 2 * half + cc;          // 32-column chunk of the stage
                float d[32];
                tmem_ld32(tmem + 128 * u + (static_cast<uint32_t>(32 * quad) << 16) + 32 * c, d);
                // columns 8pc..8pc+7 of the chunk: 32-byte piece pc ^ (rr mod 4)
                uint8_t* rowp = stg + c * kDtBox + rr * 128;
                float4 s4[8];
#pragma unroll
                for (int pc = 0; pc < 8; ++pc)
                  s4[pc] = *reinterpret_cast<const float4*>(rowp + (((pc >> 1) ^ (rr & 3)) << 5) + (pc & 1) * 16);
                tmem_wait_ld();
#pragma unroll
                for (int pc = 0; pc < 8; ++pc) {
                  float4 x = s4[pc];
                  x.x = fmaf(gT, x.x, d[4 * pc]);
                  x.y = fmaf(gT, x.y, d[4 * pc + 1]);
                  x.z = fmaf(gT, x.z, d[4 * pc + 2]);
                  x.w = fmaf(gT, x.w, d[4 * pc + 3]);
                  *reinterpret_cast<float4*>(rowp + (((pc >> 1) ^ (rr & 3)) << 5) + (pc & 1) * 16) = x;
                }
              }
            } else {
              ok = false;
            }
            tc_fence_before();
            fence_proxy_async_smem();
            // the 4 warps of this set (both column halves) meet before the store
            if (set == 0)
              asm volatile("bar.sync 3, 128;" ::: "memory");
            else
              asm volatile("bar.sync 4, 128;" ::: "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive(&du_free[u]);
            if (store_leader && ok && !*abort_flag) {
              for (int c = 0; c < 4; ++c)
                tma_store_2d(&tmS, stg + c * kDtBox, 128 * b + 32 * c, item * p.dk + 64 * q);
              tma_store_commit();
              if (b == nb - 1 && mb == nm - 1) {
                pend_st = st;      // its store reads while the outputs are formed
              } else {
                tma_store_wait_read();
                mbar_arrive(&empty[st]);
              }
            }
          }
        }
      }
      // outputs: o_t[c] = O^T[c][t] + sum_{j<=t} A[t][j] v_j[c]; warps of column half
      // `half` take the blocks b = half, half + 2, ...
      const bool go = wall(ok && mbar_wait(do_full, nitem & 1, abort_flag, p.err));
      if (go) {
        tc_fence_after();
        for (int b = half; b < nb; b += 2) {
          float ot[16];
          tmem_ld16(tmem + 256 + 16 * b + (static_cast<uint32_t>(32 * quad) << 16), ot);
          tmem_wait_ld();
          const int c = 128 * b + 32 * quad + lane;     // d_v column
          float vj[kDtMaxT];                             // v_j[c], rows from Tn on are zero
#pragma unroll
          for (int j = 0; j < kDtMaxT; ++j)
            vj[j] = *reinterpret_cast<const float*>(vb + (c >> 5) * kDtChunk + sw32_off(j, c));
#pragma unroll
          for (int t = 0; t < kDtMaxT; ++t) {
            if (t >= p.Tn) break;
            float s = ot[t];
#pragma unroll
            for (int j = 0; j <= t; ++j) s = fmaf(att[t * kDtMaxT + j], vj[j], s);
            const size_t oi = ((static_cast<size_t>(n) * p.Tn + t) * p.H + h) * p.dv + c;
            if (p.o_bf16)
              static_cast<__nv_bfloat16*>(p.o)[oi] = __float2bfloat16_rn(s);
            else
              static_cast<float*>(p.o)[oi] = s;
          }
        }
      } else {
        ok = false;
      }
      if (pend_st >= 0) {
        tma_store_wait_read();
        mbar_arrive(&empty[pend_st]);
        pend_st = -1;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(do_free);
      // every worker is done with this item's tiles before the next item's are formed
      asm volatile("bar.sync 2, 256;" ::: "memory");
    }
    if (store_leader) tma_store_wait_all();   // the store issuers
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// The driver's tensor-map encoder, looked up once (thread-safe static init).
PFN_cuTensorMapEncodeTiled_v12000 dt_encode_fn() {
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    return nullptr;
  }();
  return fn;
}

}  // namespace

bool decode_steps_tc_supported(int Tn, int dk, int dv) {
  return Tn >= 1 && Tn <= kDtMaxT && (dk == 128 || dk == 256) && dv % 128 == 0 &&
         DtLayout(dk, dv).smem <= 232448 &&
         static_cast<uint32_t>(Tn * (2 * dk + dv) * 2) <= kDtStage;
}

// The tensor cores pay off once the 2 Tn FMAs per state element dominate the
// pass: from 12 tokens on (the CUDA-core kernel is HBM-bound below that).
bool decode_steps_tc_preferred(int Tn, int dk, int dv) {
  return Tn >= 12 && decode_steps_tc_supported(Tn, dk, dv);
}

cudaError_t launch_decode_steps_tc(const void* q, const void* k, const void* v, float* state,
                                   void* o, DType o_t, int N, int Tn, int H, int dk, int dv,
                                   const HeadDecay& dec, unsigned* err, cudaStream_t s) {
  if (!decode_steps_tc_supported(Tn, dk, dv)) return cudaErrorNotSupported;
  const long long items = static_cast<long long>(N) * H;
  if (items * dk >= (1ll << 31)) return cudaErrorNotSupported;
  auto fn = dt_encode_fn();
  if (!fn) return cudaErrorNotSupported;
  // the state as [N*H*dk rows][dv] float32, boxes of 32 columns x 64 rows
  CUtensorMap mS;
  cuuint64_t gdim[2] = {static_cast<cuuint64_t>(dv), static_cast<cuuint64_t>(N) * H * dk};
  cuuint64_t gstride[1] = {static_cast<cuuint64_t>(dv) * 4};
  cuuint32_t box[2] = {32, 64};
  cuuint32_t estr[2] = {1, 1};
  if (fn(&mS, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, state, gdim, gstride, box, estr,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorNotSupported;
  // q, k: [N*Tn rows][H*dk] bf16, boxes of dk x Tn; v: [N*Tn][H*dv], boxes of 128 x Tn
  CUtensorMap mQ, mK, mV;
  {
    const cuuint32_t one[2] = {1, 1};
    cuuint64_t gq[2] = {static_cast<cuuint64_t>(H) * dk, static_cast<cuuint64_t>(N) * Tn};
    cuuint64_t sq[1] = {static_cast<cuuint64_t>(H) * dk * 2};
    cuuint32_t bq[2] = {static_cast<cuuint32_t>(dk), static_cast<cuuint32_t>(Tn)};
    cuuint64_t gv[2] = {static_cast<cuuint64_t>(H) * dv, static_cast<cuuint64_t>(N) * Tn};
    cuuint64_t sv[1] = {static_cast<cuuint64_t>(H) * dv * 2};
    cuuint32_t bv[2] = {128, static_cast<cuuint32_t>(Tn)};
    if (fn(&mQ, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(q), gq, sq, bq, one,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS ||
        fn(&mK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(k), gq, sq, bq, one,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS ||
        fn(&mV, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(v), gv, sv, bv, one,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorNotSupported;
  }
  DecTcParams p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.o = o;
  p.o_bf16 = o_t == DType::BF16 ? 1 : 0;
  p.nitems = static_cast<int>(items);
  p.Tn = Tn;
  p.H = H;
  p.dk = dk;
  p.dv = dv;
  p.dec = dec;
  p.err = err;
  const size_t smem = DtLayout(dk, dv).smem;
  cudaError_t e = cudaFuncSetAttribute(decode_multi_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int grid = p.nitems < sms ? p.nitems : sms;
  decode_multi_tc_kernel<<<grid, kDtThreads, smem, s>>>(mS, mQ, mK, mV, p);
  return cudaGetLastError();
}

}  // namespace ret

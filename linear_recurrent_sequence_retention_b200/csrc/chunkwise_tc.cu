// Chunkwise retention forward on tcgen05 tensor cores (bf16 in, f32 accumulate).
//
// The chunkwise form (abeam.tech summary of Sun et al. 2023, section
// 「長文の学習にはチャンク再帰を使う」): inside a chunk of L tokens the parallel
// form; across chunks a decayed read of the state carried from the previous
// chunk; at the chunk end the state is updated.  Row i of chunk c:
//     O[i] = sum_{j<=i} gamma^(i-j) (q_i.k_j) v_j  +  gamma^(i+1) q_i S_(c-1)
//     S_c  = gamma^L S_(c-1) + sum_j gamma^(L-1-j) k_j^T v_j
//
// Two warp-specialised kernels (warp 0: TMA producer, warp 1: TMEM
// allocation + MMA issue, warps 2..9: two warpgroups that own the 128 TMEM
// lanes):
//
//  state_kernel   one CTA per (sequence, head, 128 rows of d_k, NS columns of
//                 d_v).  The state block lives in TMEM (f32) for the whole
//                 sequence, in two accumulators used in turn: the MMA
//                 accumulates a chunk's contribution dS = (zeta K)_hi^T V +
//                 (zeta K)_lo^T V into one (zeta_j = gamma^(L-1-j); warpgroup
//                 B turns every staged K tile into zeta*K hi/lo tiles ahead of
//                 it) while the other holds the state entering the chunk;
//                 warpgroup A then forms S = gamma^L S_prev + dS in place,
//                 releases the older accumulator to the next chunk and stores
//                 S in the next chunk's workspace slot (as a hi/lo bf16 pair)
//                 while that chunk runs.  The final f32 state goes to
//                 state_out.
//
//  output_kernel  persistent, one CTA per SM, each CTA owning an NV-wide part
//                 of d_v (the halves of d_v = 512 form a 2-CTA cluster that
//                 exchanges the GroupNorm statistics through distributed
//                 shared memory) and walking output tiles (chunk, 128-row
//                 block r of the chunk, head).  MMA order per tile:
//                   O  = Q S_hi + Q S_lo           (then O *= gamma^(i+1) in TMEM)
//                   Sc = Q K_kb^T  for kb = 0..r   (double-buffered in TMEM)
//                   O  += P_hi V_kb + P_lo V_kb    (P = decayed, masked Sc, kept
//                                                   in TMEM as the MMA's A operand)
//                 O and the score buffers swap TMEM halves from tile to tile,
//                 so the next tile's Q S MMAs run during this tile's
//                 GroupNorm + gate epilogue.  Each epilogue warpgroup forms P
//                 for half of the keys and owns half of the output columns.
//
// Precision: q, k, v enter the MMAs as the exact bf16 values they are; the
// three rounded intermediates (decayed scores, carried state, zeta*K) enter as
// hi + lo bf16 pairs (about 16 significant bits), so the result carries
// f32-accumulation error only.  All tiles are loaded by TMA (no multicast)
// into 128-byte-swizzled shared memory; every wait is bounded (tc_ptx.cuh)
// and on expiry the CTA drains its in-flight copies and MMAs, frees TMEM and
// returns.
#include <cudaTypedefs.h>

#include <cstring>

#include "launch.h"
#include "tc_ptx.cuh"

namespace ret {
namespace {

using namespace tc;

constexpr int kRowsPerTile = 128;     // MMA M, TMEM lanes, query rows per CTA
constexpr int kKeysPerBlock = 128;    // keys per score tile
constexpr int kThreads = 320;         // 10 warps
constexpr int kWgThreads = 128;       // one warpgroup
constexpr uint32_t kBox = 8192;       // one [64 rows][128 B] box
constexpr uint32_t kTallBox = 16384;  // one [128 rows][128 B] box

struct SeqInfo {
  int s, c, a, b, cs, len;   // sequence, chunk, sequence [a,b), chunk start, chunk length
};

// chunk slot -> (sequence, chunk); false if the slot holds no chunk
__device__ __forceinline__ bool slot_to_chunk(const SeqLayout& L, const int32_t* chunk_base,
                                              long long slot, SeqInfo& si) {
  if (L.cu == nullptr) {
    const int nch = ceil_div(L.T, L.chunk);
    si.s = static_cast<int>(slot / nch);
    si.c = static_cast<int>(slot % nch);
    if (si.s >= L.nseq) return false;
  } else {
    if (slot >= chunk_base[L.nseq]) return false;
    int lo = 0, hi = L.nseq - 1;               // largest s with chunk_base[s] <= slot
    while (lo < hi) {
      int mid = (lo + hi + 1) >> 1;
      if (chunk_base[mid] <= slot) lo = mid; else hi = mid - 1;
    }
    si.s = lo;
    si.c = static_cast<int>(slot - chunk_base[lo]);
  }
  seq_bounds(L, si.s, si.a, si.b);
  si.cs = si.a + si.c * L.chunk;
  si.len = min(L.chunk, si.b - si.cs);
  return si.len > 0;
}

// AND of `v` over the 32 lanes of the warp (tcgen05.ld/st are warp-collective,
// so every guard around them must be warp-uniform).
__device__ __forceinline__ bool warp_all(bool v) { return __all_sync(0xffffffffu, v) != 0; }

// Named barrier over the 256 threads of warps 2..9.
__device__ __forceinline__ void wg2_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

// Named barrier over the 128 threads of epilogue warpgroup wg (warps 2+4wg .. 5+4wg).
__device__ __forceinline__ void wg_sync(int wg) {
  if (wg == 0) asm volatile("bar.sync 2, 128;" ::: "memory");
  else asm volatile("bar.sync 3, 128;" ::: "memory");
}

// AND of `v` over the 128 threads of warps 2..5 (named barrier 2); every one of
// them gets the same answer, so loops that contain barrier 2 stay uniform.
__device__ __forceinline__ bool wga_all(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 2, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(v ? 1u : 0u)
      : "memory");
  return r != 0;
}

// ===========================================================================
// State kernel
// ===========================================================================
constexpr int kStTok = 64;           // tokens per pipeline stage
constexpr int kStThreads = 480;      // 15 warps: producer, MMA, warpgroup A, two converter
                                     // warpgroups, the store warp of the fp16 copy of v
constexpr int kCvtThreads = 256;     // the converter warps 6..13

struct StateParams {
  SeqLayout L;
  const int32_t* chunk_base;
  const int32_t* order;              // varlen: sequences longest first (else nullptr)
  const float* state_in;
  float* state_out;
  int H, dk, dv;
  int write_v16;                     // store the fp16 copy of v (the d_k blocks split its columns)
  // anti-causal mode: the chunks are walked last to first and each carries the
  // state of everything after it, F_(c-1) = gamma^L F_c + sum_j gamma^(j+1) k_j^T v_j
  int anti;
  HeadDecay dec;
  unsigned* err;
};

template <int NS>
struct StCfg {
  static constexpr uint32_t kKBytes = 2 * kBox;              // 64 tokens x 128 rows of d_k
  static constexpr uint32_t kVBytes = (NS / 64) * kBox;      // 64 tokens x NS
  static constexpr uint32_t kStage = kKBytes + kVBytes;      // zeta*K | V, both fp16 in place
  // staging for the TMA stores of the state entering a chunk: two 128 x 64
  // fp16 boxes, filled in turn
  static constexpr uint32_t kStaging = 2 * kTallBox;
  static constexpr int kStagesFit = static_cast<int>((232448 - kStaging - 1024) / kStage);
  static constexpr int kStages = kStagesFit < 6 ? kStagesFit : 6;
  static constexpr uint32_t kOffStaging = kStages * kStage;
  static constexpr uint32_t kSmem = kOffStaging + kStaging + 256;
};

template <int NS>
__global__ void __launch_bounds__(kStThreads, 1)
state_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
             const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmV16,
             const StateParams p) {
  using SC = StCfg<NS>;
  constexpr int NSTG = SC::kStages;
  constexpr uint32_t kStage = SC::kStage;
  constexpr uint32_t kKBytes = SC::kKBytes;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* staging = smem + SC::kOffStaging;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SC::kOffStaging + SC::kStaging);
  uint64_t* full = bars;
  uint64_t* empty = full + NSTG;
  uint64_t* kready = empty + NSTG;
  uint64_t* acc_free = kready + NSTG;    // warpgroup A has read the older accumulator
  uint64_t* acc_full = acc_free + 1;     // the chunk's contribution is complete
  uint64_t* drain = acc_full + 1;
  uint32_t* tmem_hold = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_hold + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // 1-D grid, sequence-major: all (head, d_k block, d_v part) CTAs of a
  // sequence are adjacent, and packed sequences go longest first
  const int mblocks = (p.dk + 127) / 128;        // 128-row blocks of d_k (d_k = 64: one, half used)
  const int zn = mblocks * (p.dv / NS);
  const int rank = static_cast<int>(blockIdx.x / (p.H * zn));
  const int rem = static_cast<int>(blockIdx.x % (p.H * zn));
  const int h = rem / zn, zz = rem % zn;
  const int s = p.order ? p.order[rank] : rank;
  const int m = zz % mblocks, part = zz / mblocks;
  const int kboxes = p.dk >= 128 ? 2 : 1;        // 64-column K boxes loaded per stage
  // the fp16 copy of this CTA's value columns leaves from the V stages; the d_k
  // blocks of a column part split its 64-column boxes, so no CTA of the pair
  // holds its stages longer than the other
  const int v16_per = ((NS / 64) + mblocks - 1) / mblocks;    // boxes stored per d_k block
  const int v16_b0 = m * v16_per, v16_b1 = min((m + 1) * v16_per, NS / 64);
  const bool v16_out = p.write_v16 && v16_b0 < v16_b1;
  const SeqLayout& L = p.L;
  int a, b;
  seq_bounds(L, s, a, b);
  const int nch = ceil_div(b - a, L.chunk);
  const Decay1 dec(p.dec, h);
  // the chunk taken c-th: chunk c, or chunk nch-1-c in the anti-causal mode
  auto chunk_of = [&](int c) { return p.anti ? nch - 1 - c : c; };

  if (threadIdx.x == 0) {
    for (int i = 0; i < NSTG; ++i) {
      mbar_init(&full[i], 1);
      // released by the MMA, and by the copy store once it has read the stage
      mbar_init(&empty[i], v16_out ? 2 : 1);
      mbar_init(&kready[i], kCvtThreads);
    }
    mbar_init(acc_free, kWgThreads);
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    if ((smem_u32(smem) & 1023u) != 0) {
      *abort_flag = 1;
      raise_error(p.err, kErrTimeout);
    }
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_hold, 2 * NS);       // two accumulators of NS columns
    tmem_relinquish();
  }
  if (kboxes == 1) {
    // d_k = 64: the second 64-row half of every zeta*K tile stays zero, so the
    // 128-row MMA adds nothing to TMEM rows 64..127
    for (int st = 0; st < NSTG; ++st)
      for (int o = threadIdx.x * 16; o < static_cast<int>(kBox); o += kStThreads * 16)
        *reinterpret_cast<uint4*>(smem + st * kStage + kBox + o) = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_hold;

  if (warp == 0) {
    // ---------------- TMA producer: K rows and V rows (bf16) ----------------
    if (lane == 0 && !*abort_flag) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int it = 0;
      bool ok = true;
      for (int c = 0; c < nch && ok; ++c) {
        const int tok0 = a + chunk_of(c) * L.chunk;
        const int Lc = min(L.chunk, b - tok0);
        for (int sb = 0; sb * kStTok < Lc; ++sb, ++it) {
          const int st = it % NSTG;
          if (!mbar_wait(&empty[st], ((it / NSTG) & 1) ^ 1, abort_flag, p.err)) { ok = false; break; }
          uint8_t* base = smem + st * kStage;
          mbar_arrive_expect_tx(&full[st], kboxes * kBox + SC::kVBytes);
          const int y = tok0 + sb * kStTok;
          for (int bx = 0; bx < kboxes; ++bx)
            tma_load_2d(base + bx * kBox, &tmK, &full[st], h * p.dk + 128 * m + 64 * bx, y);
          for (int bx = 0; bx < NS / 64; ++bx)
            tma_load_2d(base + kKBytes + bx * kBox, &tmV, &full[st],
                        h * p.dv + NS * part + 64 * bx, y);
        }
      }
      if (!ok) {   // drain: the last load issued into each stage must land before exit
        for (int j = 1; j <= NSTG && it - j >= 0; ++j) {
          const int i2 = it - j;
          mbar_wait_drain(&full[i2 % NSTG], (i2 / NSTG) & 1);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer: dS_c = (zeta K)^T V, fp16 operands ----------------
    // into accumulator c & 1 (the other one holds the state entering the chunk)
    if (lane == 0 && !*abort_flag) {
      constexpr uint32_t idesc = idesc_f16_f32(128, NS, true, true);
      int it = 0;
      bool ok = true, issued = false;
      for (int c = 0; c < nch && ok; ++c) {
        const int Lc = min(L.chunk, b - (a + chunk_of(c) * L.chunk));
        const uint32_t acc = tmem + (c & 1) * NS;
        // this accumulator last held S_(c-2), which warpgroup A has read by now
        if (c > 0 && !mbar_wait(acc_free, (c - 1) & 1, abort_flag, p.err)) { ok = false; break; }
        tc_fence_after();
        for (int sb = 0; sb * kStTok < Lc; ++sb, ++it) {
          const int st = it % NSTG;
          if (!mbar_wait(&kready[st], (it / NSTG) & 1, abort_flag, p.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t zk = smem_u32(smem + st * kStage);
          const uint32_t vb = zk + kKBytes;
#pragma unroll
          for (int ks = 0; ks < kStTok / 16; ++ks)
            mma_bf16(acc, sdesc_sw128(zk + ks * 2048, kBox, 1024), sdesc_sw128(vb + ks * 2048, kBox, 1024),
                     idesc, (sb | ks) != 0);
          issued = true;
          mma_commit(&empty[st]);
        }
        if (ok) mma_commit(acc_full);
      }
      if (!ok && issued) {
        mma_commit(drain);
        mbar_wait_drain(drain, 0);
      }
    }
  } else if (warp < 6) {
    // ---------------- warpgroup A: the carried state ----------------
    // S_(c-1) sits in accumulator (c+1) & 1 while the MMA accumulates the
    // chunk's contribution dS_c into accumulator c & 1; then
    //     S_c = gamma^L S_(c-1) + dS_c   (written over dS_c)
    // releases the older accumulator for chunk c+1, and S_c (the state entering
    // chunk c+1) goes to that chunk's workspace slot, as fp16, while chunk c+1
    // runs.
    const int quad = warp & 3;
    const int row = quad * 32 + lane;            // TMEM lane = row of the state block
    const int i = 128 * m + row;                 // d_k index
    const bool row_ok = i < p.dk;                // d_k = 64: TMEM rows 64..127 hold zeros
    const uint32_t trow = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const size_t st_off = ((static_cast<size_t>(s) * p.H + h) * p.dk + (row_ok ? i : 0)) * p.dv + NS * part;
    const bool leader = threadIdx.x == 64;
    if (leader) tma_prefetch_desc(&tmW);
    bool range_ok = true;
    auto slot_of = [&](int c) -> long long {
      return L.cu == nullptr ? static_cast<long long>(s) * ceil_div(L.T, L.chunk) + c
                             : static_cast<long long>(p.chunk_base[s]) + c;
    };
    // The state in accumulator column `col` -> workspace slot `slot` as fp16,
    // one 128 x 64 box per TMA store, through the two staging boxes in turn.
    // Barrier 2 is reached by all 128 threads the same number of times.
    int nbox = 0;
    auto stage_state = [&](uint32_t col, long long slot) {
      const bool slot_ok = slot >= 0 && slot < L.nslots;
      // workspace rows of this CTA's 128 d_k rows
      const int wrow = static_cast<int>(((slot_ok ? slot : 0) * p.H + h) * p.dk) + 128 * m;
#pragma unroll 1
      for (int j = 0; j < NS / 32; j += 2, ++nbox) {
        uint8_t* box = staging + (nbox & 1) * kTallBox;
        float r[2][32];
        tmem_ld32(trow + col + 32 * j, r[0]);
        tmem_ld32(trow + col + 32 * (j + 1), r[1]);
        tmem_wait_ld();
        // this staging box is free once the store issued from it two boxes ago
        // has read it (at most the other box's store is still pending)
        if (leader) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
        asm volatile("bar.sync 2, 128;" ::: "memory");
        // row `row` of a 128 x 64 swizzled box: 16-byte piece cc of the row
        // goes to piece cc ^ (row & 7)
        float amax = 0.f;
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) {
          const float* x = &r[cc >> 2][(cc & 3) * 8];
#pragma unroll
          for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(x[e]));
          const uint4 u = make_uint4(pack_f16(x[0], x[1]), pack_f16(x[2], x[3]),
                                     pack_f16(x[4], x[5]), pack_f16(x[6], x[7]));
          *reinterpret_cast<uint4*>(box + row * 128 + ((cc ^ (row & 7)) << 4)) = u;
        }
        range_ok = range_ok && !(amax > kF16Max);    // NaN passes here; it is not a range event
        fence_proxy_async_smem();
        asm volatile("bar.sync 2, 128;" ::: "memory");
        if (leader && slot_ok) {
          // a box of min(d_k, 128) rows: the first rows of the staged box
          tma_store_2d(&tmW, box, NS * part + 32 * j, wrow);
          tma_store_commit();
        }
      }
    };
    bool ok = wga_all(!*abort_flag);
    if (ok && nch > 0) {
      // the state entering chunk 0 (state_in, or zero) into accumulator 1
#pragma unroll 1
      for (int j = 0; j < NS / 32; ++j) {
        float r[32];
        if (p.state_in && row_ok) {
          const float4* src = reinterpret_cast<const float4*>(p.state_in + st_off + 32 * j);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float4 x = src[e];
            r[4 * e] = x.x; r[4 * e + 1] = x.y; r[4 * e + 2] = x.z; r[4 * e + 3] = x.w;
          }
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) r[e] = 0.f;
        }
        tmem_st32(trow + NS + 32 * j, r);
      }
      tmem_wait_st();
      stage_state(NS, slot_of(chunk_of(0)));
    }
    for (int c = 0; c < nch && ok; ++c) {
      const int Lc = min(L.chunk, b - (a + chunk_of(c) * L.chunk));
      ok = wga_all(mbar_wait(acc_full, c & 1, abort_flag, p.err));
      if (!ok) break;
      tc_fence_after();
      const uint32_t dcol = (c & 1) * NS, pcol = ((c + 1) & 1) * NS;
      const float gL = dec.pow(Lc);
      const uint64_t gL2 = f2_make(gL, gL);
#pragma unroll 1
      for (int j = 0; j < NS / 32; ++j) {
        float sp[32], sd[32];
        tmem_ld32(trow + pcol + 32 * j, sp);
        tmem_ld32(trow + dcol + 32 * j, sd);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const uint64_t v2 = f2_fma(f2_make(sp[e], sp[e + 1]), gL2, f2_make(sd[e], sd[e + 1]));
          sd[e] = f2_lo(v2);
          sd[e + 1] = f2_hi(v2);
        }
        tmem_st32(trow + dcol + 32 * j, sd);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(acc_free);                     // accumulator pcol may take chunk c+1
      if (c + 1 < nch) stage_state(dcol, slot_of(chunk_of(c + 1)));
    }
    if (leader) tma_store_wait_all();
    if (!range_ok) raise_error(p.err, kErrRange);
    // final state: S_(nch-1), in accumulator (nch-1) & 1
    if (ok && nch > 0) {
      if (p.state_out) {
        const uint32_t fcol = ((nch - 1) & 1) * NS;
        for (int j = 0; j < NS / 32; ++j) {
          float r[32];
          tmem_ld32(trow + fcol + 32 * j, r);
          tmem_wait_ld();
          if (!row_ok) continue;
          float4* dst = reinterpret_cast<float4*>(p.state_out + st_off + 32 * j);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            dst[e] = make_float4(r[4 * e], r[4 * e + 1], r[4 * e + 2], r[4 * e + 3]);
        }
      }
    } else if (ok && p.state_out && row_ok) {   // empty sequence: the state passes through
      for (int j = 0; j < NS; j += 4) {
        float4 x = p.state_in ? *reinterpret_cast<const float4*>(p.state_in + st_off + j)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
        *reinterpret_cast<float4*>(p.state_out + st_off + j) = x;
      }
    }
  } else if (warp < 14) {
    // ---------------- converter warps 6..13: the fp16 MMA operands, ahead of the MMA ----------------
    // K rows -> zeta*K (fp16, in place; thread u owns half a row), V rows ->
    // fp16 (in place; thread u owns row u).
    const int u = threadIdx.x - 192;              // 0..255
    constexpr int kVRows = (NS / 64) * 64;        // V rows of a stage: (NS/64) boxes x 64 tokens
    const int krow = u >> 1, khalf = u & 1;       // this thread's K row (box krow/64) and half
    const bool k_mine = krow < 64 * kboxes;
    int it = 0;
    bool ok = !*abort_flag, range_ok = true;
    for (int c = 0; c < nch && ok; ++c) {
      const int tok0 = a + chunk_of(c) * L.chunk;
      const int Lc = min(L.chunk, b - tok0);
      for (int sb = 0; sb * kStTok < Lc; ++sb, ++it) {
        const int st = it % NSTG;
        if (!mbar_wait(&full[st], (it / NSTG) & 1, abort_flag, p.err)) { ok = false; break; }
        uint8_t* stage = smem + st * kStage;
        if (k_mine) {
          // zeta*K, pieces 4*khalf .. 4*khalf+3 of row krow%64 of box krow/64:
          // zeta_j = gamma^(L-1-j), or gamma^(j+1) in the anti-causal mode
          const int jtok = sb * kStTok + (krow & 63);
          const float z = jtok < Lc ? dec.pow(p.anti ? jtok + 1 : Lc - 1 - jtok) : 0.f;
          uint4* rp = reinterpret_cast<uint4*>(stage + (krow >> 6) * kBox + (krow & 63) * 128);
          const int sw = krow & 7;
          uint4 w4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) w4[e] = rp[(4 * khalf + e) ^ sw];
          const uint64_t z2 = f2_make(z, z);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const uint32_t w[4] = {w4[e].x, w4[e].y, w4[e].z, w4[e].w};
            uint32_t wh[4];
#pragma unroll
            for (int q2 = 0; q2 < 4; ++q2) {
              const uint64_t p2 = f2_mul(f2_make(bf16_lo(w[q2]), bf16_hi(w[q2])), z2);
              wh[q2] = pack_f16(f2_lo(p2), f2_hi(p2));
            }
            rp[(4 * khalf + e) ^ sw] = make_uint4(wh[0], wh[1], wh[2], wh[3]);
          }
        }
        if (u < kVRows) {
          // V row u: box u/64, token row u%64, converted bf16 -> fp16
          uint4* rp = reinterpret_cast<uint4*>(stage + kKBytes + u * 128);
          // every piece converts the same way, so visit them in the order
          // e ^ (row & 7): 8 consecutive rows then touch 8 different bank groups
          const int sw = u & 7;
          uint4 w4[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) w4[e] = rp[e ^ sw];
          uint32_t amax = 0;                              // largest |bf16| bit pattern, per half
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const uint32_t w[4] = {w4[e].x, w4[e].y, w4[e].z, w4[e].w};
#pragma unroll
            for (int q2 = 0; q2 < 4; ++q2) amax = __vmaxu2(amax, w[q2] & 0x7fff7fffu);
            rp[e ^ sw] = make_uint4(bf16x2_to_f16x2(w[0]), bf16x2_to_f16x2(w[1]),
                                    bf16x2_to_f16x2(w[2]), bf16x2_to_f16x2(w[3]));
          }
          // |v| >= 2^16 (bf16 0x4780) has no fp16 value; rows past the
          // sequence's end hold other tokens (or the zero fill) and are not
          // this sequence's to report
          const uint32_t big = max(amax & 0xffffu, amax >> 16);
          const int jtok = sb * kStTok + (u & 63);
          if (big >= 0x4780u && jtok < Lc) range_ok = false;
        }
        fence_proxy_async_smem();
        mbar_arrive(&kready[st]);
      }
    }
    if (!range_ok) raise_error(p.err, kErrRange);
  } else if (warp == 14) {
    // ---------------- store warp: the fp16 copy of v ----------------
    // Each stage's converted V rows go out by TMA store as soon as the
    // converters are done; the stage returns to the producer once the store
    // has read it (its second arrival on `empty`, beside the MMA's).
    if (v16_out && lane == 0 && !*abort_flag) {
      tma_prefetch_desc(&tmV16);
      int it = 0;
      bool ok = true;
      for (int c = 0; c < nch && ok; ++c) {
        const int tok0 = a + chunk_of(c) * L.chunk;
        const int Lc = min(L.chunk, b - tok0);
        for (int sb = 0; sb * kStTok < Lc; ++sb, ++it) {
          const int st = it % NSTG;
          if (!mbar_wait(&kready[st], (it / NSTG) & 1, abort_flag, p.err)) { ok = false; break; }
          const int y = tok0 + sb * kStTok;
          uint8_t* stage = smem + st * kStage;
          for (int bx = v16_b0; bx < v16_b1; ++bx)
            tma_store_2d(&tmV16, stage + kKBytes + bx * kBox, h * p.dv + NS * part + 64 * bx, y);
          tma_store_commit();
          tma_store_wait_read();
          mbar_arrive(&empty[st]);
        }
      }
      tma_store_wait_all();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * NS);
  }
}

// ===========================================================================
// Output kernel (persistent)
// ===========================================================================
constexpr uint32_t kOutStage = 32768;

struct OutParams {
  SeqLayout L;
  const int32_t* chunk_base;
  bool has_state_in;
  void* out;
  int out_bf16;
  const void* g;
  int g_bf16;
  const float* gn_w;
  const float* gn_b;
  float eps;
  int gated;
  int g_tma;                   // gate tile streamed by TMA (bf16 gate)
  int y_tma;                   // full output tiles written by TMA (bf16 output)
  int acc_out;                 // float32 output, ungated: out += o instead of out = o
  // anti-causal mode: o_i = sum_{j >= i} gamma^(j-i) (q_i . k_j) v_j + gamma^(L-1-i) q_i F,
  // F the state of everything after the chunk (the state pass's anti-causal walk)
  int anti;
  // the carried state read transposed (s_kmajor): the slots hold another
  // pass's state [dv rows][stored columns]; this pass multiplies by the
  // columns s_col0 .. s_col0+dk-1 of it, as a K-major operand
  int s_kmajor, s_col0;
  // dynamic tile order (dyn): each cluster takes its next tile from a global
  // counter (zeroed before the launch), in the static order's sequence of
  // tiles; the fetch is made once per cluster and handed to every role
  int dyn;         // selects the kernel instantiation (set on the host)
  int* tile_ctr;
  int H, dk, dv;
  int rb;                      // 128-row blocks per chunk
  int parts;                   // d_v parts (cluster size)
  int ntiles;                  // chunk slots x heads x row blocks (persistent kernel)
  int nch;                     // chunks per sequence (equal-length layout)
  int nclusters;               // clusters in the persistent grid
  int shift;                   // per-round rotation of the tile order (persistent kernel)
  HeadDecay dec;
  unsigned* err;
};

template <int DK, int NV>
struct OutCfg {
  static constexpr uint32_t kQBytes = (DK / 64) * kTallBox;
  // barriers | gamma^d table | GroupNorm pairs passed between the two
  // warpgroups | GroupNorm pairs received from the partner CTA
  static constexpr uint32_t kMiscBytes = 256 + 512 + 1024 + 1024;
  // Everything but Q and the small tables is ring: the loads in flight per SM
  // set the pace of this kernel (a tile moves ~0.5 MB from L2).  The
  // gate/output tile (NV/64 boxes of 128 rows x 64 columns, two per stage)
  // takes ring stages too, loaded after the tile's other units and released
  // by the epilogue once its stores have read them.
  static constexpr int kStages =
      static_cast<int>((232448 - kQBytes - kMiscBytes) / kOutStage);
  static constexpr int kGateStages =
      static_cast<int>(((NV / 64) * kTallBox + kOutStage - 1) / kOutStage);
  static_assert(kStages >= kGateStages + 2, "the ring must hold the gate tile and a key unit");
  static_assert(2 * kStages + 14 <= 32, "barrier area");
  static constexpr uint32_t kOffStages = kQBytes;
  static constexpr uint32_t kOffMisc = kOffStages + kStages * kOutStage;
  static constexpr uint32_t kSmem = kOffMisc + kMiscBytes;
  // TMEM (fixed): O in columns [0, NV), score buffers 0 and 1 in [256, 384)
  // and [384, 512).  P of key piece j (keys 32j..32j+31) is written as fp16
  // over the first 16 of that piece's own 32 score columns (two keys per
  // column); the decayed query rows that read the carried state (d_k values,
  // two per column) take a whole score buffer.
  static constexpr uint32_t kColSB = 256;
};


// One 128-row output tile: rows 128r..128r+127 of a chunk, one head, all d_v
// columns of this CTA's part.
struct OutTile {
  SeqInfo si;
  long long slot;
  int h, r, t0, nrows;
  int kb0, nkb;                // key blocks kb0 .. kb0+nkb-1 (0..r causal, r..last anti-causal)
  bool inter;                  // reads the state carried into the chunk
};

// The tiles of one cluster.  Tile u = ((slot * H + h) * rb + (rb - 1 - r)):
// the row blocks of a (chunk, head) are adjacent, heaviest first.  In round k
// cluster c takes tile k * nclusters + (c + k * shift) mod nclusters, so each
// round covers a contiguous range of tiles (the row blocks of a chunk run at
// the same time and share its K, V and state tiles in L2) while the row block,
// and with it the tile's cost, rotates from round to round for every cluster.
// Every role of both CTAs of the cluster walks the same sequence.
struct TileWalk {
  int k = 0;   // static order: rounds taken
  int n = 0;   // dynamic order: tiles taken from the cluster's queue
  // Tile u of the fixed tile sequence; false if it holds no rows.
  __device__ __forceinline__ bool decode(const OutParams& p, int u, OutTile& t) const {
    // 32-bit index arithmetic: the host keeps the tile count below 2^31
    const unsigned gh = static_cast<unsigned>(u) / static_cast<unsigned>(p.rb);
    const unsigned slot = gh / static_cast<unsigned>(p.H);
    t.h = static_cast<int>(gh - slot * static_cast<unsigned>(p.H));
    // heaviest row block first: the last one (causal) or the first (anti-causal)
    const int rr = static_cast<int>(static_cast<unsigned>(u) - gh * static_cast<unsigned>(p.rb));
    t.r = p.anti ? rr : p.rb - 1 - rr;
    t.slot = slot;
    if (p.L.cu == nullptr) {
      const unsigned sq = slot / static_cast<unsigned>(p.nch);
      if (static_cast<int>(sq) >= p.L.nseq) return false;
      t.si.s = static_cast<int>(sq);
      t.si.c = static_cast<int>(slot - sq * static_cast<unsigned>(p.nch));
      t.si.a = t.si.s * p.L.T;
      t.si.b = t.si.a + p.L.T;
      t.si.cs = t.si.a + t.si.c * p.L.chunk;
      t.si.len = min(p.L.chunk, t.si.b - t.si.cs);
      if (t.si.len <= 0) return false;
    } else if (!slot_to_chunk(p.L, p.chunk_base, slot, t.si)) {
      return false;
    }
    if (t.r * kRowsPerTile >= t.si.len) return false;
    t.t0 = t.si.cs + t.r * kRowsPerTile;
    t.nrows = min(kRowsPerTile, t.si.len - t.r * kRowsPerTile);
    if (p.anti) {
      t.kb0 = t.r;
      t.nkb = (t.si.len + kKeysPerBlock - 1) / kKeysPerBlock - t.r;
      t.inter = t.si.cs + t.si.len < t.si.b || p.has_state_in;   // a later chunk, or a state in
    } else {
      t.kb0 = 0;
      t.nkb = t.r + 1;
      t.inter = t.si.c > 0 || p.has_state_in;
    }
    return true;
  }
  // The static order: in round k cluster c takes tile k * nclusters + (c + k * shift) mod nclusters.
  __device__ __forceinline__ bool next(const OutParams& p, int cid, OutTile& t) {
    while (true) {
      const int base = k * p.nclusters;
      if (base >= p.ntiles) return false;
      const int u = base + static_cast<int>(static_cast<unsigned>(cid + k * p.shift) %
                                            static_cast<unsigned>(p.nclusters));
      ++k;
      if (u < p.ntiles && decode(p, u, t)) return true;
    }
  }
};

// AND of `v` over the 256 epilogue threads (named barrier 4); every one of them
// gets the same answer.
__device__ __forceinline__ bool epi_all(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 4, 256, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(v ? 1u : 0u)
      : "memory");
  return r != 0;
}

template <int DK, int NV, bool DYN>
__global__ void __launch_bounds__(kThreads, 1)
output_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmS,
              const __grid_constant__ CUtensorMap tmG, const __grid_constant__ CUtensorMap tmY,
              const OutParams p) {
  using C = OutCfg<DK, NV>;
  constexpr int NST = C::kStages;
  constexpr int kHalf = NV / 2;                       // O columns per epilogue warpgroup
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffMisc);
  uint64_t* full = bars;                 // [NST] stage loaded
  uint64_t* empty = full + NST;          // [NST] stage consumed
  uint64_t* bar_q = empty + NST;         // Q tile loaded
  uint64_t* q_free = bar_q + 1;          // every MMA and every epilogue read of Q is done
  uint64_t* bar_s = q_free + 1;          // [2] scores ready in TMEM
  uint64_t* bar_p = bar_s + 2;           // [2] P written over the scores
  uint64_t* pv_done = bar_p + 2;         // [2] the P V MMAs of a score buffer are done
  uint64_t* bar_pp = pv_done + 2;        // decayed query rows written (state read operand)
  uint64_t* bar_o = bar_pp + 1;          // all MMAs of the tile done
  uint64_t* drain = bar_o + 1;
  uint64_t* bar_x = drain + 1;           // the partner's statistics have arrived
  uint64_t* bar_xack = bar_x + 1;        // the partner has read this CTA's statistics
  uint32_t* tmem_hold = reinterpret_cast<uint32_t*>(bar_xack + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_hold + 1);
  float* pow_tab = reinterpret_cast<float*>(smem + C::kOffMisc + 256);    // gamma^d, d < 128
  float* wgx = reinterpret_cast<float*>(smem + C::kOffMisc + 768);        // [128][2]
  float* xrecv = reinterpret_cast<float*>(smem + C::kOffMisc + 1792);     // [128][2]
  // dynamic tile queue (ungated launches only, in place of xrecv): kDynQ tile
  // indices, their full barriers (arrived by the fetcher) and, in the first
  // CTA of the cluster, their empty barriers (arrived by every other role)
  constexpr int kDynQ = 4;
  int* dq = reinterpret_cast<int*>(smem + C::kOffMisc + 1792);
  uint64_t* dq_full = reinterpret_cast<uint64_t*>(smem + C::kOffMisc + 1792 + 64);
  uint64_t* dq_empty = dq_full + kDynQ;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int part = blockIdx.x % p.parts;
  const int cid = blockIdx.x / p.parts;
  const bool xchg = p.parts > 1 && p.gated;           // GroupNorm spans both CTAs of the cluster
  // K(kb) is kKU units of kKB 64-column boxes (128 keys each)
  constexpr int kKU = DK >= 128 ? DK / 128 : 1;
  constexpr int kKB = DK >= 128 ? 2 : 1;
  // the gate/output tile: NV/64 boxes of 128 rows x 64 columns in kGateStages
  // ring stages (two boxes per stage)
  constexpr int kIoBoxes = NV / 64;
  constexpr int kGS = C::kGateStages;
  constexpr int kBoxesPerStage = static_cast<int>(kOutStage / kTallBox);
  // ring units of one tile before its gate stages
  auto tile_units = [&](const OutTile& tt) {
    return tt.nkb * (kKU + 2) + (tt.inter ? DK / 64 : 0);
  };
  auto io_staged = [&](const OutTile& t) {
    return (p.gated && p.g_tma) || (p.y_tma && t.nrows == kRowsPerTile);
  };

  if (threadIdx.x == 0) {
    for (int i = 0; i < NST; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(bar_q, 1);
    mbar_init(q_free, 1 + 2 * kWgThreads);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_s[i], 1);
      mbar_init(&bar_p[i], 2 * kWgThreads);
      mbar_init(&pv_done[i], 1);
    }
    mbar_init(bar_pp, 2 * kWgThreads);
    mbar_init(bar_o, 1);
    mbar_init(drain, 1);
    mbar_init(bar_x, 1);                  // armed per tile with the partner's 1 KB
    mbar_init(bar_xack, kWgThreads);
    if (DYN && !p.gated) {
      for (int i = 0; i < kDynQ; ++i) {
        mbar_init(&dq_full[i], 1);
        mbar_init(&dq_empty[i], 2 + 3 * (p.parts - 1));
      }
    }
    *abort_flag = 0;
    if ((smem_u32(smem) & 1023u) != 0) {
      *abort_flag = 1;
      raise_error(p.err, kErrTimeout);
    }
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_hold, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_hold;
  const bool dynq = DYN && !p.gated;    // the dynamic queue lives where xrecv would
  const bool cl = p.parts > 1 && (p.gated || dynq);
  if (cl) cluster_arrive_relaxed();      // barrier initialisation done (waited on before first use)
  bool cluster_waited = false;           // this thread has passed that first cluster barrier phase

  TileWalk walk;
  OutTile t;
  const bool fetcher = cluster_ctarank() == 0;   // the cluster's first CTA fetches the tiles
  // The next tile in the dynamic order, for one thread of a role: the fetcher
  // (the first CTA's producer) takes it from the counter and publishes it;
  // every other role waits for it. Returns the tile index (-1 at the end);
  // *okr = false if a wait ran out.
  auto dyn_take = [&](bool fetch, bool* okr) -> int {
    const int slot = walk.n % kDynQ;
    const uint32_t ph = (walk.n / kDynQ) & 1;
    if (cl && !cluster_waited) {
      cluster_wait();                    // the partner's barriers are initialised
      cluster_waited = true;
    }
    int u = -1;
    if (fetch) {
      if (!mbar_wait(&dq_empty[slot], ph ^ 1, abort_flag, p.err)) { *okr = false; return -1; }
      OutTile tt;
      do {
        u = atomicAdd(p.tile_ctr, 1);
      } while (u < p.ntiles && !walk.decode(p, u, tt));
      if (u >= p.ntiles) u = -1;
      dq[slot] = u;
      if (p.parts > 1) {
        st_cluster_f32(cluster_addr(&dq[slot], 1u), __int_as_float(u));
        mbar_arrive_cluster(cluster_addr(&dq_full[slot], 1u));
      }
      mbar_arrive(&dq_full[slot]);
    } else {
      if (!mbar_wait_cluster(&dq_full[slot], ph, abort_flag, p.err)) { *okr = false; return -1; }
      u = dq[slot];
    }
    ++walk.n;
    return u;
  };
  // a consumer role is done reading the queue slot it took last
  auto dyn_release = [&]() {
    const int slot = (walk.n - 1) % kDynQ;
    if (fetcher) mbar_arrive(&dq_empty[slot]);
    else mbar_arrive_cluster(cluster_addr(&dq_empty[slot], 0u));
  };

  // Per tile, the ring units in the order the MMA consumes them (32 KB each):
  //   K(0), then for kb = 0..r: [K(kb+1) if kb < r], V(kb) keys 0-63, V(kb) keys 64-127
  //   (fp16 copy of v), then [S of d_k rows 64u..64u+63, u < DK/64 (fp16), if
  //   the chunk reads a state].  The gate tile goes to its own buffer.
  // The ring runs on across tiles, so the next tile's first key blocks stream
  // in during this tile's epilogue.
  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0 && !*abort_flag) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmS);
      if (p.gated && p.g_tma) tma_prefetch_desc(&tmG);
      int it = 0, tq = 0;
      bool ok = true;
      auto next = [&](uint32_t bytes) -> uint8_t* {
        const int st = it % NST;
        if (!mbar_wait(&empty[st], ((it / NST) & 1) ^ 1, abort_flag, p.err)) return nullptr;
        mbar_arrive_expect_tx(&full[st], bytes);
        return smem + C::kOffStages + st * kOutStage;
      };
      while (ok) {
        if (dynq) {
          const int u = dyn_take(fetcher, &ok);
          if (u < 0) break;
          if (!fetcher) dyn_release();
          walk.decode(p, u, t);
        } else if (!walk.next(p, cid, t)) {
          break;
        }
        // Q of this tile, once the previous tile's MMAs and epilogue are done with Q
        if (tq > 0 && !mbar_wait(q_free, (tq - 1) & 1, abort_flag, p.err)) { ok = false; break; }
        mbar_arrive_expect_tx(bar_q, C::kQBytes);
        for (int u = 0; u < DK / 64; ++u)
          tma_load_2d(smem + u * kTallBox, &tmQ, bar_q, t.h * DK + 64 * u, t.t0);
        ++tq;
        auto load_k = [&](int kb) {
          for (int ku = 0; ku < kKU && ok; ++ku) {
            uint8_t* dst = next(kKB * kTallBox);
            if (!dst) { ok = false; break; }
            for (int bx = 0; bx < kKB; ++bx)
              tma_load_2d(dst + bx * kTallBox, &tmK, &full[it % NST], t.h * DK + 128 * ku + 64 * bx,
                          t.si.cs + kKeysPerBlock * kb);
            ++it;
          }
        };
        auto load_v = [&](int kb) {
          for (int vu = 0; vu < 2 && ok; ++vu) {
            uint8_t* dst = next((NV / 64) * kBox);
            if (!dst) { ok = false; break; }
            for (int bx = 0; bx < NV / 64; ++bx)
              tma_load_2d(dst + bx * kBox, &tmV, &full[it % NST], t.h * p.dv + NV * part + 64 * bx,
                          t.si.cs + kKeysPerBlock * kb + 64 * vu);
            ++it;
          }
        };
        load_k(t.kb0);
        for (int kk = 0; kk < t.nkb && ok; ++kk) {
          if (kk + 1 < t.nkb) load_k(t.kb0 + kk + 1);
          load_v(t.kb0 + kk);
        }
        if (ok && t.inter) {
          for (int u = 0; u < DK / 64 && ok; ++u) {
            uint8_t* dst = next((NV / 64) * kBox);
            if (!dst) { ok = false; break; }
            if (p.s_kmajor) {
              // 64 state rows of this pass = 64 columns of the stored state, all NV of its rows
              tma_load_2d(dst, &tmS, &full[it % NST], p.s_col0 + 64 * u,
                          static_cast<int>((t.slot * p.H + t.h) * NV));
            } else {
              const int srow = static_cast<int>((t.slot * p.H + t.h) * DK) + 64 * u;
              for (int bx = 0; bx < NV / 64; ++bx)
                tma_load_2d(dst + bx * kBox, &tmS, &full[it % NST], NV * part + 64 * bx, srow);
            }
            ++it;
          }
        }
        if (ok && io_staged(t)) {
          // the gate/output tile (or, ungated, just the stages its bf16
          // output is staged in: an arrival with no bytes)
          const bool load_g = p.gated && p.g_tma;
          for (int gs = 0; gs < kGS && ok; ++gs) {
            const int nbx = min(kIoBoxes - kBoxesPerStage * gs, kBoxesPerStage);
            uint8_t* dst = next(load_g ? nbx * kTallBox : 0);
            if (!dst) { ok = false; break; }
            if (load_g)
              for (int bb = 0; bb < nbx; ++bb)
                tma_load_2d(dst + bb * kTallBox, &tmG, &full[it % NST],
                            t.h * p.dv + NV * part + 64 * (kBoxesPerStage * gs + bb), t.t0);
            ++it;
          }
        }
      }
      if (!ok) {
        // let the copies already issued land before the CTA can exit
        if (tq > 0) mbar_wait_drain(bar_q, (tq - 1) & 1);
        for (int j = 1; j <= NST && it - j >= 0; ++j) {
          const int i2 = it - j;
          mbar_wait_drain(&full[i2 % NST], (i2 / NST) & 1);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    // Per tile:  Sc(0), Sc(1);  for kb: [P(kb)] O (+)= P(kb) V(kb), Sc(kb+2);
    // then [decayed Q rows] O += Qd S.  The first P V of a tile overwrites O:
    // its P is formed only after the epilogue has finished with the previous
    // tile's O.
    if (lane == 0 && !*abort_flag) {
      constexpr uint32_t id_qk = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t id_pv = idesc_f16_f32(128, NV, false, true);
      constexpr uint32_t id_qs_k = idesc_f16_f32(128, NV, false, false);   // K-major state
      const uint32_t q_base = smem_u32(smem);
      const uint32_t st_base = smem_u32(smem + C::kOffStages);
      const uint32_t sbuf0 = tmem + C::kColSB;
      int it = 0, tq = 0, sblk = 0, npp = 0;   // npp: tiles that read a carried state
      bool ok = true, issued = false;
      auto stage_wait = [&]() -> uint32_t {
        const int st = it % NST;
        if (!mbar_wait(&full[st], (it / NST) & 1, abort_flag, p.err)) return 0;
        tc_fence_after();
        return st_base + st * kOutStage;
      };
      auto stage_free = [&]() {
        mma_commit(&empty[it % NST]);
        ++it;
      };
      while (ok) {
        if (dynq) {
          const int u = dyn_take(false, &ok);
          if (u < 0) break;
          dyn_release();
          walk.decode(p, u, t);
        } else if (!walk.next(p, cid, t)) {
          break;
        }
        if (!mbar_wait(bar_q, tq & 1, abort_flag, p.err)) { ok = false; break; }
        tc_fence_after();
        auto issue_qk = [&](int kb) -> bool {          // kb: the tile's kb-th key block
          const uint32_t dst = sbuf0 + 128 * (kb & 1);
          for (int ku = 0; ku < kKU; ++ku) {
            const uint32_t sb = stage_wait();
            if (!sb) return false;
#pragma unroll
            for (int kk = 0; kk < 4 * kKB; ++kk) {
              const int qbox = ku * 2 + kk / 4;
              mma_bf16(dst, sdesc_sw128(q_base + qbox * kTallBox + (kk & 3) * 32, 16, 1024),
                       sdesc_sw128(sb + (kk / 4) * kTallBox + (kk & 3) * 32, 16, 1024), id_qk,
                       (ku | kk) != 0);
            }
            issued = true;
            stage_free();
          }
          mma_commit(&bar_s[(sblk + kb) & 1]);
          if (kb == t.nkb - 1) mma_commit(q_free);     // the MMAs are done with Q
          return true;
        };
        if (!issue_qk(0)) { ok = false; break; }
        if (t.nkb >= 2 && !issue_qk(1)) { ok = false; break; }
        for (int kb = 0; kb < t.nkb && ok; ++kb) {
          const int sg = sblk + kb;
          if (!mbar_wait(&bar_p[sg & 1], (sg >> 1) & 1, abort_flag, p.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t pbuf = sbuf0 + 128 * (kb & 1);
          for (int vu = 0; vu < 2; ++vu) {
            const uint32_t sb = stage_wait();
            if (!sb) { ok = false; break; }
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const int ks = vu * 4 + kk;                      // keys 16ks .. 16ks+15
              mma_bf16_ts(tmem, pbuf + 32 * (ks >> 1) + 8 * (ks & 1),
                          sdesc_sw128(sb + kk * 2048, kBox, 1024), id_pv, kb > 0 || ks > 0);
            }
            stage_free();
          }
          if (!ok) break;
          mma_commit(&pv_done[sg & 1]);
          // the next scores go to the buffer this P V has just been issued from
          // (tcgen05 MMAs of one thread execute in issue order)
          if (kb + 2 < t.nkb && !issue_qk(kb + 2)) { ok = false; break; }
        }
        if (!ok) break;
        if (t.inter) {
          // O += (gamma^(i+1) q_i) S: the decayed query rows (fp16, in the score
          // buffer after the last one used) times the carried state (fp16)
          if (!mbar_wait(bar_pp, npp & 1, abort_flag, p.err)) { ok = false; break; }
          ++npp;
          tc_fence_after();
          const uint32_t abuf = sbuf0 + 128 * (t.nkb & 1);
          for (int u = 0; u < DK / 64 && ok; ++u) {
            const uint32_t sb = stage_wait();
            if (!sb) { ok = false; break; }
            if (p.s_kmajor) {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_bf16_ts(tmem, abuf + 32 * u + 8 * kk, sdesc_sw128(sb + kk * 32, 16, 1024),
                            id_qs_k, true);
            } else {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_bf16_ts(tmem, abuf + 32 * u + 8 * kk, sdesc_sw128(sb + kk * 2048, kBox, 1024),
                            id_pv, true);
            }
            stage_free();
          }
          if (!ok) break;
        }
        mma_commit(bar_o);
        if (io_staged(t)) {
          // The gate stages belong to the epilogue, but this thread still waits
          // for them to land: its waits then stay in ring order, so a later
          // wait on one of these stages cannot match the parity of the phase
          // one lap older while the gate load is still in flight.
          for (int gs = 0; gs < kGS && ok; ++gs, ++it)
            ok = mbar_wait(&full[it % NST], (it / NST) & 1, abort_flag, p.err);
          if (!ok) break;
        }
        sblk += t.nkb;
        ++tq;
      }
      if (!ok && issued) {
        mma_commit(drain);
        mbar_wait_drain(drain, 0);
      }
    }
  } else {
    // ---------------- epilogue: warpgroup wg owns key pieces 2wg, 2wg+1, d_k
    // columns [wg*DK/2, (wg+1)*DK/2) of the decayed query rows, and O columns
    // [wg*NV/2, (wg+1)*NV/2) ----------------
    const int wg = (warp - 2) >> 2;                   // 0 or 1
    const int quad = warp & 3;
    const int row = quad * 32 + lane;                 // query row within the block
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t o_cols = tmem + lane_off + wg * kHalf;
    const uint32_t sbuf0 = tmem + lane_off + C::kColSB;
    const int et = threadIdx.x - 64;                  // 0..255
    const bool wg_leader = (et & 127) == 0;           // first thread of the warpgroup
    constexpr bool kBoxPerWg = kHalf >= 64;           // each warpgroup owns whole boxes
    const uint32_t other = xchg ? (cluster_ctarank() ^ 1u) : 0u;
    int tq = 0, sblk = 0, git = 0;                    // git: ring position, as the producer counts
    bool ok = true;
    float pmax = 0.f;                                 // largest |P| and |decayed q| formed
    while (true) {
      int u = 0;
      bool got = true;
      if (dynq) {
        bool wok = true;
        u = dyn_take(false, &wok);
        got = warp_all(wok);
      } else {
        got = walk.next(p, cid, t);              // the same for every thread
        u = got ? 0 : -1;
        got = true;
      }
      // uniform over the 256 epilogue threads: the named barriers below stay matched
      if (!epi_all(got && ok && !*abort_flag)) break;
      if (u < 0) break;                          // every thread read the same index
      if (dynq) {
        if (et == 0) dyn_release();              // all 256 threads have read the slot
        walk.decode(p, u, t);
      }
      const int r = t.r;
      const int i = r * kRowsPerTile + row;            // row within the chunk
      const bool staged = io_staged(t);
      const int g0 = git + tile_units(t);              // this tile's first gate stage
      git = g0 + (staged ? kGS : 0);
      auto io_box = [&](int bx) -> uint8_t* {
        return smem + C::kOffStages + ((g0 + bx / kBoxesPerStage) % NST) * kOutStage +
               (bx % kBoxesPerStage) * kTallBox;
      };
      const Decay1 dec(p.dec, t.h);
      // gamma^d for this tile's head (the previous tile's P is complete: every
      // epilogue thread passed the barrier in epi_all above after forming it)
      if (et < 128) pow_tab[et] = dec.pow(et);
      wg2_sync();
      for (int kk = 0; kk < t.nkb && ok; ++kk) {
        const int kb = t.kb0 + kk;                       // key block within the chunk
        const int sg = sblk + kk;
        if (!warp_all(mbar_wait(&bar_s[sg & 1], (sg >> 1) & 1, abort_flag, p.err))) { ok = false; break; }
        tc_fence_after();
        const bool diag = kb == r;
        // off-diagonal: gamma^(i-j) = gamma^(i - 128kb - 127) * gamma^(127 - j'), or in
        // the anti-causal mode gamma^(j-i) = gamma^(128kb - i) * gamma^(j')
        const float arow = diag ? 0.f
                                : dec.pow(p.anti ? kKeysPerBlock * kb - i : i - kKeysPerBlock * kb - 127);
        const int key_lim = t.si.len - kKeysPerBlock * kb;   // keys j' >= key_lim are past the chunk
        const uint32_t buf = sbuf0 + 128 * (kk & 1);
#pragma unroll 1
        for (int j = 2 * wg; j < 2 * wg + 2; ++j) {
          float x[32];
          tmem_ld32(buf + 32 * j, x);
          float wv[32];
          if (diag && p.anti) {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const int jp = 32 * j + e;
              wv[e] = jp >= row ? pow_tab[jp - row] : 0.f;
            }
          } else if (diag) {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const int jp = 32 * j + e;
              wv[e] = jp <= row ? pow_tab[row - jp] : 0.f;
            }
          } else if (p.anti) {
            // gamma^(32j + e), read as float4 from the table in ascending order
#pragma unroll
            for (int m4 = 0; m4 < 8; ++m4) {
              const float4 t4 = *reinterpret_cast<const float4*>(pow_tab + 32 * j + 4 * m4);
              wv[4 * m4] = t4.x * arow; wv[4 * m4 + 1] = t4.y * arow;
              wv[4 * m4 + 2] = t4.z * arow; wv[4 * m4 + 3] = t4.w * arow;
            }
          } else {
            // gamma^(127 - 32j - e), read as float4 from the table in descending order
            const uint64_t a2 = f2_make(arow, arow);
#pragma unroll
            for (int m = 0; m < 8; ++m) {
              const float4 t4 = *reinterpret_cast<const float4*>(pow_tab + 124 - 32 * j - 4 * m);
              const uint64_t w0 = f2_mul(f2_make(t4.w, t4.z), a2);
              const uint64_t w1 = f2_mul(f2_make(t4.y, t4.x), a2);
              wv[4 * m] = f2_lo(w0); wv[4 * m + 1] = f2_hi(w0);
              wv[4 * m + 2] = f2_lo(w1); wv[4 * m + 3] = f2_hi(w1);
            }
          }
          if (key_lim < 32 * j + 32) {
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (32 * j + e >= key_lim) wv[e] = 0.f;
          }
          tmem_wait_ld();
          uint32_t pw[16];
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const uint64_t p2 = f2_mul(f2_make(x[e], x[e + 1]), f2_make(wv[e], wv[e + 1]));
            pmax = fmaxf(pmax, fmaxf(fabsf(f2_lo(p2)), fabsf(f2_hi(p2))));
            pw[e >> 1] = pack_f16(f2_lo(p2), f2_hi(p2));
          }
          tmem_st16(buf + 32 * j, pw);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bar_p[sg & 1]);
      }
      if (t.inter && ok) {
        // the decayed query rows gamma^(i+1) q_i (fp16) into the score buffer
        // after the last one used, once the P V MMAs that read it are done
        if (t.nkb >= 2) {
          const int sg = sblk + t.nkb - 2;
          ok = warp_all(mbar_wait(&pv_done[sg & 1], (sg >> 1) & 1, abort_flag, p.err));
          if (ok) tc_fence_after();
        }
        // the Q tile's TMA writes are visible to this thread's loads (Q is not
        // reloaded before this thread releases it through q_free)
        if (ok) ok = warp_all(mbar_wait(bar_q, tq & 1, abort_flag, p.err));
        if (ok) {
          // gamma^(i+1), or gamma^(L-1-i) in the anti-causal mode (rows past the chunk: 0)
          const float sc = p.anti ? (i < t.si.len ? dec.pow(t.si.len - 1 - i) : 0.f) : dec.pow(i + 1);
          const uint64_t sc2 = f2_make(sc, sc);
          const uint32_t abuf = sbuf0 + 128 * (t.nkb & 1);
          // this warpgroup's d_k columns: half-box pieces of 32 values
#pragma unroll 1
          for (int c0 = wg * (DK / 2); c0 < (wg + 1) * (DK / 2); c0 += 32) {
            const uint8_t* qrow = smem + (c0 >> 6) * kTallBox + row * 128;
            const int pc0 = (c0 & 63) >> 3;            // first 16-byte piece of the 32 values
            uint32_t pw[16];
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
              const uint4 u = *reinterpret_cast<const uint4*>(qrow + (((pc0 + c4) ^ (row & 7)) << 4));
              const uint32_t wq[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
              for (int q2 = 0; q2 < 4; ++q2) {
                const uint64_t d2 = f2_mul(f2_make(bf16_lo(wq[q2]), bf16_hi(wq[q2])), sc2);
                pmax = fmaxf(pmax, fmaxf(fabsf(f2_lo(d2)), fabsf(f2_hi(d2))));
                pw[4 * c4 + q2] = pack_f16(f2_lo(d2), f2_hi(d2));
              }
            }
            tmem_st16(abuf + (c0 >> 1), pw);
          }
          tmem_wait_st();
          tc_fence_before();
        }
        mbar_arrive(bar_pp);
      }
      mbar_arrive(q_free);                             // this thread is done reading Q
      sblk += t.nkb;
      ok = warp_all(ok && mbar_wait(bar_o, tq & 1, abort_flag, p.err));
      if (ok) tc_fence_after();
      // GroupNorm statistics in one pass: sums of (x - x0) and (x - x0)^2 with
      // x0 the row's first value in this warpgroup's half (a shift that keeps
      // the sums well conditioned).  Warpgroup 1 hands its (mean, M2) to
      // warpgroup 0, which combines the halves, exchanges with the partner
      // CTA (the other d_v part) and hands back (mean, 1/std).  Barriers and
      // the exchange are unconditional, so an aborted CTA still meets its
      // partner.
      float mean_all = 0.f, rstd = 0.f;
      if (p.gated) {
        float mean_w = 0.f, m2_w = 0.f;
        if (ok) {
          uint64_t s1 = 0, s2 = 0;
          float x0 = 0.f;
          for (int j = 0; j < kHalf / 32; ++j) {
            float x[32];
            tmem_ld32(o_cols + 32 * j, x);
            tmem_wait_ld();
            if (j == 0) x0 = x[0];
            const uint64_t nx0 = f2_make(-x0, -x0);
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const uint64_t d = f2_add(f2_make(x[e], x[e + 1]), nx0);
              s1 = f2_add(s1, d);
              s2 = f2_fma(d, d, s2);
            }
          }
          const float S1 = f2_lo(s1) + f2_hi(s1), S2 = f2_lo(s2) + f2_hi(s2);
          mean_w = x0 + S1 * (1.0f / kHalf);
          m2_w = fmaxf(S2 - S1 * S1 * (1.0f / kHalf), 0.f);
        }
        if (wg == 1) {
          wgx[2 * row] = mean_w;
          wgx[2 * row + 1] = m2_w;
        }
        wg2_sync();
        if (wg == 0) {
          const float m1 = wgx[2 * row], m21 = wgx[2 * row + 1];
          const float dd = m1 - mean_w;
          float mean = 0.5f * (mean_w + m1);
          float m2 = m2_w + m21 + dd * dd * (0.5f * kHalf);
          float cnt = static_cast<float>(NV);
          if (xchg) {
            // the other d_v part: once the partner has read the previous
            // pair, send this part's (mean, M2) into its receive buffer with
            // st.async (the store signals 8 bytes on the partner's barrier,
            // which its first epilogue thread arms for 128 rows), then read
            // the partner's pair and release this CTA's receive buffer
            if (!cluster_waited) {
              cluster_wait();                        // partner's barriers are initialised
              cluster_waited = true;
            }
            bool xok = tq == 0 || mbar_wait_cluster(bar_xack, (tq - 1) & 1, abort_flag, p.err);
            if (et == 0) mbar_arrive_expect_tx(bar_x, kWgThreads * 8);
            st_async_f32x2(cluster_addr(&xrecv[2 * row], other), mean, m2, cluster_addr(bar_x, other));
            xok = mbar_wait_cluster(bar_x, tq & 1, abort_flag, p.err) && xok;
            if (xok) {
              const float mo = xrecv[2 * row], m2o = xrecv[2 * row + 1];
              const float d = mo - mean;
              m2 = m2 + m2o + d * d * (cnt * 0.5f);
              mean = 0.5f * (mean + mo);
              cnt *= 2.f;
            } else {
              ok = false;
            }
            mbar_arrive_cluster(cluster_addr(bar_xack, other));
          }
          mean_all = mean;
          rstd = 1.0f / sqrtf(m2 / cnt + p.eps);
          wgx[2 * row] = mean_all;
          wgx[2 * row + 1] = rstd;
        }
        wg2_sync();
        if (wg == 1) {
          mean_all = wgx[2 * row];
          rstd = wgx[2 * row + 1];
        }
      }

      // ---------------- GroupNorm, gate, store ----------------
      // Full tiles with a bf16 output go through shared memory (in place of the
      // gate tile, same swizzled layout) and TMA stores, one per 64-column box
      // as soon as its warpgroup has written it; partial tiles are written
      // directly so that no row past the chunk is touched.
      const bool out_tma = p.y_tma && t.nrows == kRowsPerTile;
      const bool live = row < t.nrows;
      const int col0 = NV * part + wg * kHalf;          // first d_v column of this warpgroup
      const size_t obase = (static_cast<size_t>(t.t0 + row) * p.H + t.h) * p.dv + col0;
      const float shift = -mean_all * rstd;
      bool go = warp_all(ok && !*abort_flag);
      for (int gs = 0; gs < kGS && go && staged; ++gs)
        go = warp_all(mbar_wait(&full[(g0 + gs) % NST], ((g0 + gs) / NST) & 1, abort_flag, p.err));
      if (go) tc_fence_after();
      for (int j = 0; j < kHalf / 32; ++j) {
        // this piece's 32 columns in the staged gate/output box: box, first 16-byte piece
        const int cpart = wg * kHalf + 32 * j;
        uint8_t* brow = io_box(cpart >> 6) + row * 128;
        const int pc0 = (cpart & 63) >> 3;
        if (go) {
          float x[32];
          tmem_ld32(o_cols + 32 * j, x);
          if (p.gated) {
            float gv[32];
            if (p.g_tma) {
#pragma unroll
              for (int c4 = 0; c4 < 4; ++c4) {
                const uint4 u = *reinterpret_cast<const uint4*>(brow + (((pc0 + c4) ^ (row & 7)) << 4));
                const uint32_t wv[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int q2 = 0; q2 < 4; ++q2) {
                  gv[8 * c4 + 2 * q2] = bf16_lo(wv[q2]);
                  gv[8 * c4 + 2 * q2 + 1] = bf16_hi(wv[q2]);
                }
              }
            } else if (live) {
              const float4* gp = reinterpret_cast<const float4*>(static_cast<const float*>(p.g) + obase + 32 * j);
#pragma unroll
              for (int c4 = 0; c4 < 8; ++c4) {
                const float4 f = gp[c4];
                gv[4 * c4] = f.x; gv[4 * c4 + 1] = f.y; gv[4 * c4 + 2] = f.z; gv[4 * c4 + 3] = f.w;
              }
            } else {
#pragma unroll
              for (int e = 0; e < 32; ++e) gv[e] = 0.f;
            }
            tmem_wait_ld();
            const uint64_t rs2 = f2_make(rstd, rstd), sh2 = f2_make(shift, shift);
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const uint64_t y2 = f2_fma(f2_make(x[e], x[e + 1]), rs2, sh2);
              x[e] = f2_lo(y2);
              x[e + 1] = f2_hi(y2);
            }
            if (p.gn_w || p.gn_b) {
              const int c0 = t.h * p.dv + col0 + 32 * j;
#pragma unroll
              for (int e = 0; e < 32; ++e) {
                if (p.gn_w) x[e] *= p.gn_w[c0 + e];
                if (p.gn_b) x[e] += p.gn_b[c0 + e];
              }
            }
            // swish(g) = g sigmoid(g) = u + u tanh(u) with u = g/2 (sigmoid(g) =
            // (1 + tanh(g/2))/2): one special-function op per element
            const uint64_t half2 = f2_make(0.5f, 0.5f);
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const uint64_t u2 = f2_mul(f2_make(gv[e], gv[e + 1]), half2);
              const uint64_t s2 = f2_fma(u2, f2_make(tanh_fast(f2_lo(u2)), tanh_fast(f2_hi(u2))), u2);
              const uint64_t o2 = f2_mul(f2_make(x[e], x[e + 1]), s2);
              x[e] = f2_lo(o2);
              x[e + 1] = f2_hi(o2);
            }
          } else {
            tmem_wait_ld();
          }
          if (out_tma) {
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4)
              *reinterpret_cast<uint4*>(brow + (((pc0 + c4) ^ (row & 7)) << 4)) =
                  make_uint4(pack_bf16(x[8 * c4 + 0], x[8 * c4 + 1]), pack_bf16(x[8 * c4 + 2], x[8 * c4 + 3]),
                             pack_bf16(x[8 * c4 + 4], x[8 * c4 + 5]), pack_bf16(x[8 * c4 + 6], x[8 * c4 + 7]));
          } else if (live && p.out_bf16) {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + obase + 32 * j);
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4)
              dst[c4] = make_uint4(pack_bf16(x[8 * c4 + 0], x[8 * c4 + 1]), pack_bf16(x[8 * c4 + 2], x[8 * c4 + 3]),
                                   pack_bf16(x[8 * c4 + 4], x[8 * c4 + 5]), pack_bf16(x[8 * c4 + 6], x[8 * c4 + 7]));
          } else if (live) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + obase + 32 * j);
            if (p.acc_out) {
#pragma unroll
              for (int c4 = 0; c4 < 8; ++c4) {
                const float4 a = dst[c4];
                dst[c4] = make_float4(x[4 * c4] + a.x, x[4 * c4 + 1] + a.y, x[4 * c4 + 2] + a.z,
                                      x[4 * c4 + 3] + a.w);
              }
            } else {
#pragma unroll
              for (int c4 = 0; c4 < 8; ++c4)
                dst[c4] = make_float4(x[4 * c4], x[4 * c4 + 1], x[4 * c4 + 2], x[4 * c4 + 3]);
            }
          }
        }
        if (kBoxPerWg && out_tma && (j & 1)) {       // uniform over the warpgroup
          // box cpart/64 is complete: hand it to the TMA engine
          fence_proxy_async_smem();
          wg_sync(wg);
          if (wg_leader && go) {
            tma_store_2d(&tmY, io_box(cpart >> 6), t.h * p.dv + NV * part + 64 * (cpart >> 6), t.t0);
            tma_store_commit();
          }
        }
      }
      // every read of this tile's O is complete before this thread forms the
      // next tile's first P (which lets the MMA overwrite O)
      tc_fence_before();
      if (!kBoxPerWg && out_tma) {                   // boxes shared by both warpgroups
        fence_proxy_async_smem();
        wg2_sync();
        if (et == 0 && go) {
          for (int bx = 0; bx < kIoBoxes; ++bx)
            tma_store_2d(&tmY, io_box(bx), t.h * p.dv + NV * part + 64 * bx, t.t0);
          tma_store_commit();
        }
      }
      // the staging units go back to the producer once the stores have read
      // them (the global writes complete on their own)
      if (out_tma && go && (kBoxPerWg ? wg_leader : et == 0)) tma_store_wait_read();
      if (staged) {
        wg2_sync();
        if (et == 0)
          for (int gs = 0; gs < kGS; ++gs) mbar_arrive(&empty[(g0 + gs) % NST]);
      }
      ++tq;
    }
    if (pmax > kF16Max) raise_error(p.err, kErrRange);
  }
  if (cl) {
    if (!cluster_waited) cluster_wait();
    cluster_arrive();
    cluster_wait();        // the partner has made its last remote access here
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ===========================================================================
// Output kernel for one-block chunks (compact: two CTAs per SM)
// ===========================================================================
// When every chunk is a single 128-row block (chunk <= 128) a tile has one
// key block: a handful of MMAs against fixed costs (the Q and state loads, the
// GroupNorm/gate pass).  This variant holds half an SM: 6 warps (producer, MMA
// issuer, one epilogue warpgroup that forms P over all 128 keys and owns all
// output columns), 256 TMEM columns (O, then the score tile) and 16 KB ring
// stages in about 100 KB of shared memory, so two tiles share every SM and one
// tile's epilogue overlaps the other's loads and MMAs.  Same arithmetic as
// output_kernel (hi/lo P and state, one-pass GroupNorm statistics, one-op
// swish), for d_k <= 128 and d_v parts of <= 128 columns.
constexpr int kThreadsC = 192;
constexpr uint32_t kStageC = 16384;

template <int DK, int NV>
struct OutCfgC {
  static constexpr uint32_t kQBytes = (DK / 64) * kTallBox;
  // barriers | gamma^d table | the partner CTA's GroupNorm (mean, M2) per row
  static constexpr uint32_t kMiscBytes = 256 + 512 + 1024;
  static constexpr uint32_t kBudget = 113 * 1024;                 // two CTAs per SM
  static constexpr int kStages = static_cast<int>((kBudget - kQBytes - kMiscBytes) / kStageC);
  static constexpr uint32_t kOffStages = kQBytes;
  static constexpr uint32_t kOffMisc = kOffStages + kStages * kStageC;
  static constexpr uint32_t kSmem = kOffMisc + kMiscBytes;
  static constexpr uint32_t kTmemO = 0, kTmemS = 128;
};

// Named barrier over the 128 threads of the compact kernel's epilogue warpgroup.
__device__ __forceinline__ void epi_sync_c() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

template <int DK, int NV>
__global__ void __launch_bounds__(256, 2)   // 6 warps, registers sized as for 8 (allocation granularity)
output_kernel_c(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmS,
                const __grid_constant__ CUtensorMap tmG, const __grid_constant__ CUtensorMap tmY,
                const OutParams p) {
  using C = OutCfgC<DK, NV>;
  constexpr int NST = C::kStages;
  static_assert(DK <= 128 && NV <= 128, "compact tiles: d_k <= 128, d_v part <= 128");
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffMisc);
  uint64_t* full = bars;                 // [NST]
  uint64_t* empty = full + NST;          // [NST]
  uint64_t* bar_q = empty + NST;
  uint64_t* bar_pv = bar_q + 1;          // the P V MMAs are done (the score tile is free)
  uint64_t* bar_s = bar_pv + 1;          // scores ready in TMEM
  uint64_t* bar_p = bar_s + 1;           // P written over the scores
  uint64_t* bar_pp = bar_p + 1;          // decayed query rows written over the score tile
  uint64_t* bar_o = bar_pp + 1;          // all MMAs done
  uint64_t* drain = bar_o + 1;
  uint64_t* bar_x = drain + 1;           // the partner's statistics have arrived
  uint32_t* tmem_hold = reinterpret_cast<uint32_t*>(bar_x + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_hold + 1);
  float* pow_tab = reinterpret_cast<float*>(smem + C::kOffMisc + 256);    // gamma^d
  float* xrecv = reinterpret_cast<float*>(smem + C::kOffMisc + 768);     // [128][2]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int part = blockIdx.x % p.parts;
  const long long slot = blockIdx.x / p.parts;
  const int h = blockIdx.y;
  SeqInfo si;
  // Identical for both CTAs of a cluster, so a skipped slot skips together.
  if (slot >= p.L.nslots) return;
  if (!slot_to_chunk(p.L, p.chunk_base, slot, si)) return;
  const int t0 = si.cs;                                   // first token of the chunk
  const int nrows = min(kRowsPerTile, si.len);
  const bool need_inter = si.c > 0 || p.has_state_in;
  const bool xchg = p.parts > 1 && p.gated;
  const Decay1 dec(p.dec, h);
  // ring units (16 KB): K (DK/64 boxes of 128 keys x 64 d_k), V (keys 0-63,
  // 64-127; fp16 copy), [S of d_k rows 64u..64u+63 (fp16)], then the
  // gate/output tile, one 128 x 64 box per unit
  const int n_mma_units = DK / 64 + 2 + (need_inter ? DK / 64 : 0);
  auto io_box = [&](int bx) -> uint8_t* {
    return smem + C::kOffStages + ((n_mma_units + bx) % NST) * kStageC;
  };

  if (threadIdx.x == 0) {
    for (int i = 0; i < NST; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(bar_q, 1);
    mbar_init(bar_pv, 1);
    mbar_init(bar_s, 1);
    mbar_init(bar_p, kWgThreads);
    mbar_init(bar_pp, kWgThreads);
    mbar_init(bar_o, 1);
    mbar_init(drain, 1);
    mbar_init(bar_x, kWgThreads);
    *abort_flag = 0;
    if ((smem_u32(smem) & 1023u) != 0) {
      *abort_flag = 1;
      raise_error(p.err, kErrTimeout);
    }
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_hold, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_hold;
  if (xchg) cluster_arrive_relaxed();    // barrier initialisation done (waited on before first use)

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0 && !*abort_flag) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmS);
      mbar_arrive_expect_tx(bar_q, C::kQBytes);
      for (int u = 0; u < DK / 64; ++u)
        tma_load_2d(smem + u * kTallBox, &tmQ, bar_q, h * DK + 64 * u, t0);
      int it = 0;
      bool ok = true;
      auto next = [&](uint32_t bytes) -> uint8_t* {
        const int st = it % NST;
        if (!mbar_wait(&empty[st], ((it / NST) & 1) ^ 1, abort_flag, p.err)) return nullptr;
        mbar_arrive_expect_tx(&full[st], bytes);
        return smem + C::kOffStages + st * kStageC;
      };
      for (int ku = 0; ku < DK / 64 && ok; ++ku) {
        uint8_t* dst = next(kTallBox);
        if (!dst) { ok = false; break; }
        tma_load_2d(dst, &tmK, &full[it % NST], h * DK + 64 * ku, si.cs);
        ++it;
      }
      for (int vu = 0; vu < 2 && ok; ++vu) {
        uint8_t* dst = next((NV / 64) * kBox);
        if (!dst) { ok = false; break; }
        for (int bx = 0; bx < NV / 64; ++bx)
          tma_load_2d(dst + bx * kBox, &tmV, &full[it % NST], h * p.dv + NV * part + 64 * bx,
                      si.cs + 64 * vu);
        ++it;
      }
      if (need_inter) {
        for (int u = 0; u < DK / 64 && ok; ++u) {
          const int srow = static_cast<int>((slot * p.H + h) * DK) + 64 * u;
          uint8_t* dst = next((NV / 64) * kBox);
          if (!dst) { ok = false; break; }
          for (int bx = 0; bx < NV / 64; ++bx)
            tma_load_2d(dst + bx * kBox, &tmS, &full[it % NST], NV * part + 64 * bx, srow);
          ++it;
        }
      }
      if (p.gated && p.g_tma) {      // the gate rows of this tile, for the epilogue
        tma_prefetch_desc(&tmG);
        for (int u = 0; u < NV / 64 && ok; ++u) {
          uint8_t* dst = next(kTallBox);
          if (!dst) { ok = false; break; }
          tma_load_2d(dst, &tmG, &full[it % NST], h * p.dv + NV * part + 64 * u, t0);
          ++it;
        }
      }
      if (!ok) {
        mbar_wait_drain(bar_q, 0);
        for (int j = 1; j <= NST && it - j >= 0; ++j) {
          const int i2 = it - j;
          mbar_wait_drain(&full[i2 % NST], (i2 / NST) & 1);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    // Sc = Q K^T; [P] O = P V; [decayed Q rows, written over the score tile
    // once P V is done] O += Qd S.
    if (lane == 0 && !*abort_flag) {
      constexpr uint32_t id_qk = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t id_pv = idesc_f16_f32(128, NV, false, true);
      const uint32_t q_base = smem_u32(smem);
      const uint32_t st_base = smem_u32(smem + C::kOffStages);
      int it = 0;
      bool ok = true, issued = false;
      auto stage_wait = [&]() -> uint32_t {
        const int st = it % NST;
        if (!mbar_wait(&full[st], (it / NST) & 1, abort_flag, p.err)) return 0;
        tc_fence_after();
        return st_base + st * kStageC;
      };
      auto stage_free = [&]() {
        mma_commit(&empty[it % NST]);
        ++it;
      };
      ok = mbar_wait(bar_q, 0, abort_flag, p.err);
      if (ok) tc_fence_after();
      // scores Q K^T of the chunk's keys
      for (int ku = 0; ku < DK / 64 && ok; ++ku) {
        const uint32_t sb = stage_wait();
        if (!sb) { ok = false; break; }
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16(tmem + C::kTmemS, sdesc_sw128(q_base + ku * kTallBox + kk * 32, 16, 1024),
                   sdesc_sw128(sb + kk * 32, 16, 1024), id_qk, (ku | kk) != 0);
        issued = true;
        stage_free();
      }
      if (ok) mma_commit(bar_s);
      if (ok && !mbar_wait(bar_p, 0, abort_flag, p.err)) ok = false;
      if (ok) {
        tc_fence_after();
        const uint32_t pbuf = tmem + C::kTmemS;
        for (int vu = 0; vu < 2 && ok; ++vu) {
          const uint32_t sb = stage_wait();
          if (!sb) { ok = false; break; }
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const int ks = vu * 4 + kk;                      // keys 16ks .. 16ks+15
            mma_bf16_ts(tmem + C::kTmemO, pbuf + 32 * (ks >> 1) + 8 * (ks & 1),
                        sdesc_sw128(sb + kk * 2048, kBox, 1024), id_pv, ks > 0);
          }
          stage_free();
        }
        if (ok) mma_commit(bar_pv);
      }
      if (ok && need_inter) {
        // O += (gamma^(i+1) q_i) S, the decayed query rows (fp16) over the score tile
        ok = mbar_wait(bar_pp, 0, abort_flag, p.err);
        if (ok) tc_fence_after();
        for (int u = 0; u < DK / 64 && ok; ++u) {
          const uint32_t sb = stage_wait();
          if (!sb) { ok = false; break; }
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ts(tmem + C::kTmemO, tmem + C::kTmemS + 32 * u + 8 * kk,
                        sdesc_sw128(sb + kk * 2048, kBox, 1024), id_pv, true);
          stage_free();
        }
      }
      if (ok) {
        mma_commit(bar_o);
      } else if (issued) {
        mma_commit(drain);
        mbar_wait_drain(drain, 0);
      }
    }
  } else {
    // ---------------- epilogue: one warpgroup, one thread per query row ----------------
    const int quad = warp & 3;
    const int row = quad * 32 + lane;                 // query row of the chunk
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t o_cols = tmem + lane_off + C::kTmemO;
    const int et = threadIdx.x - 64;                  // 0..127
    pow_tab[et] = dec.pow(et);
    epi_sync_c();
    bool ok = !*abort_flag;
    float pmax = 0.f;                                 // largest |P| and |decayed q| formed
    if (ok) ok = warp_all(mbar_wait(bar_s, 0, abort_flag, p.err));
    if (ok) {
      tc_fence_after();
      const uint32_t buf = tmem + lane_off + C::kTmemS;
#pragma unroll 1
      for (int j = 0; j < 4; ++j) {                   // keys 32j .. 32j+31
        float x[32];
        tmem_ld32(buf + 32 * j, x);
        float wv[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int jp = 32 * j + e;
          wv[e] = (jp <= row && jp < si.len) ? pow_tab[row - jp] : 0.f;
        }
        tmem_wait_ld();
        uint32_t pw[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const uint64_t p2 = f2_mul(f2_make(x[e], x[e + 1]), f2_make(wv[e], wv[e + 1]));
          pmax = fmaxf(pmax, fmaxf(fabsf(f2_lo(p2)), fabsf(f2_hi(p2))));
          pw[e >> 1] = pack_f16(f2_lo(p2), f2_hi(p2));
        }
        tmem_st16(buf + 32 * j, pw);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar_p);
    }
    if (ok && need_inter) {
      // the decayed query rows gamma^(row+1) q_row (fp16) over the score tile,
      // once the P V MMAs have read it
      ok = warp_all(mbar_wait(bar_pv, 0, abort_flag, p.err) && mbar_wait(bar_q, 0, abort_flag, p.err));
      if (ok) {
        tc_fence_after();
        const float sc = dec.pow(row + 1);
        const uint64_t sc2 = f2_make(sc, sc);
        const uint32_t abuf = tmem + lane_off + C::kTmemS;
#pragma unroll 1
        for (int c0 = 0; c0 < DK; c0 += 32) {
          const uint8_t* qrow = smem + (c0 >> 6) * kTallBox + row * 128;
          const int pc0 = (c0 & 63) >> 3;
          uint32_t pw[16];
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            const uint4 u = *reinterpret_cast<const uint4*>(qrow + (((pc0 + c4) ^ (row & 7)) << 4));
            const uint32_t wq[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int q2 = 0; q2 < 4; ++q2) {
              const uint64_t d2 = f2_mul(f2_make(bf16_lo(wq[q2]), bf16_hi(wq[q2])), sc2);
              pmax = fmaxf(pmax, fmaxf(fabsf(f2_lo(d2)), fabsf(f2_hi(d2))));
              pw[4 * c4 + q2] = pack_f16(f2_lo(d2), f2_hi(d2));
            }
          }
          tmem_st16(abuf + (c0 >> 1), pw);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar_pp);
      }
    }
    if (pmax > kF16Max) raise_error(p.err, kErrRange);
    if (ok) ok = mbar_wait(bar_o, 0, abort_flag, p.err);
    ok = warp_all(ok);
    if (ok) tc_fence_after();
    // GroupNorm statistics in one pass (shifted by the row's first value); the
    // two d_v parts of a cluster combine as (mean, M2) pairs through the
    // partner's receive buffer.  The exchange is unconditional, so an aborted
    // CTA still meets its partner.
    float mean_all = 0.f, rstd = 0.f;
    if (p.gated) {
      float mean = 0.f, m2 = 0.f;
      if (ok) {
        uint64_t s1 = 0, s2 = 0;
        float x0 = 0.f;
        for (int j = 0; j < NV / 32; ++j) {
          float x[32];
          tmem_ld32(o_cols + 32 * j, x);
          tmem_wait_ld();
          if (j == 0) x0 = x[0];
          const uint64_t nx0 = f2_make(-x0, -x0);
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const uint64_t d = f2_add(f2_make(x[e], x[e + 1]), nx0);
            s1 = f2_add(s1, d);
            s2 = f2_fma(d, d, s2);
          }
        }
        const float S1 = f2_lo(s1) + f2_hi(s1), S2 = f2_lo(s2) + f2_hi(s2);
        mean = x0 + S1 * (1.0f / NV);
        m2 = fmaxf(S2 - S1 * S1 * (1.0f / NV), 0.f);
      }
      float cnt = static_cast<float>(NV);
      if (xchg) {
        cluster_wait();                              // partner's barriers are initialised
        const uint32_t other = cluster_ctarank() ^ 1u;
        st_cluster_f32(cluster_addr(&xrecv[2 * row], other), mean);
        st_cluster_f32(cluster_addr(&xrecv[2 * row + 1], other), m2);
        mbar_arrive_cluster(cluster_addr(bar_x, other));
        cluster_arrive();                            // this CTA's remote accesses are done
        if (mbar_wait_cluster(bar_x, 0, abort_flag, p.err)) {
          const float mo = xrecv[2 * row], m2o = xrecv[2 * row + 1];
          const float d = mo - mean;
          m2 = m2 + m2o + d * d * (cnt * 0.5f);
          mean = 0.5f * (mean + mo);
          cnt *= 2.f;
        } else {
          ok = false;
        }
      }
      mean_all = mean;
      rstd = 1.0f / sqrtf(m2 / cnt + p.eps);
    }

    // ---------------- GroupNorm, gate, store ----------------
    const bool out_tma = p.y_tma && nrows == kRowsPerTile;
    const bool leader = threadIdx.x == 64;
    const bool live = row < nrows;
    const int col0 = NV * part;
    const size_t obase = (static_cast<size_t>(t0 + row) * p.H + h) * p.dv + col0;
    const float shift = -mean_all * rstd;
    bool go = warp_all(ok && !*abort_flag);
    if (go && p.gated && p.g_tma) {
      for (int u = 0; u < NV / 64 && go; ++u) {
        const int unit = n_mma_units + u;
        go = mbar_wait(&full[unit % NST], (unit / NST) & 1, abort_flag, p.err);
      }
      go = warp_all(go);
    }
    if (go) tc_fence_after();
    if (out_tma && leader) tma_prefetch_desc(&tmY);
    for (int j = 0; j < NV / 32; ++j) {
      uint8_t* brow = io_box(j >> 1) + row * 128;      // 64-column box j/2
      const int pc0 = (j & 1) * 4;
      if (go) {
        float x[32];
        tmem_ld32(o_cols + 32 * j, x);
        if (p.gated) {
          float gv[32];
          if (p.g_tma) {
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
              const uint4 u = *reinterpret_cast<const uint4*>(brow + (((pc0 + c4) ^ (row & 7)) << 4));
              const uint32_t wv[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
              for (int q2 = 0; q2 < 4; ++q2) {
                gv[8 * c4 + 2 * q2] = bf16_lo(wv[q2]);
                gv[8 * c4 + 2 * q2 + 1] = bf16_hi(wv[q2]);
              }
            }
          } else if (live) {
            const float4* gp = reinterpret_cast<const float4*>(static_cast<const float*>(p.g) + obase + 32 * j);
#pragma unroll
            for (int c4 = 0; c4 < 8; ++c4) {
              const float4 f = gp[c4];
              gv[4 * c4] = f.x; gv[4 * c4 + 1] = f.y; gv[4 * c4 + 2] = f.z; gv[4 * c4 + 3] = f.w;
            }
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) gv[e] = 0.f;
          }
          tmem_wait_ld();
          const uint64_t rs2 = f2_make(rstd, rstd), sh2 = f2_make(shift, shift);
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const uint64_t y2 = f2_fma(f2_make(x[e], x[e + 1]), rs2, sh2);
            x[e] = f2_lo(y2);
            x[e + 1] = f2_hi(y2);
          }
          if (p.gn_w || p.gn_b) {
            const int c0 = h * p.dv + col0 + 32 * j;
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              if (p.gn_w) x[e] *= p.gn_w[c0 + e];
              if (p.gn_b) x[e] += p.gn_b[c0 + e];
            }
          }
          // swish(g) = g sigmoid(g) = u + u tanh(u) with u = g/2: one
          // special-function op per element
          const uint64_t half2 = f2_make(0.5f, 0.5f);
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const uint64_t u2 = f2_mul(f2_make(gv[e], gv[e + 1]), half2);
            const uint64_t s2 = f2_fma(u2, f2_make(tanh_fast(f2_lo(u2)), tanh_fast(f2_hi(u2))), u2);
            const uint64_t o2 = f2_mul(f2_make(x[e], x[e + 1]), s2);
            x[e] = f2_lo(o2);
            x[e + 1] = f2_hi(o2);
          }
        } else {
          tmem_wait_ld();
        }
        if (out_tma) {
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4)
            *reinterpret_cast<uint4*>(brow + (((pc0 + c4) ^ (row & 7)) << 4)) =
                make_uint4(pack_bf16(x[8 * c4 + 0], x[8 * c4 + 1]), pack_bf16(x[8 * c4 + 2], x[8 * c4 + 3]),
                           pack_bf16(x[8 * c4 + 4], x[8 * c4 + 5]), pack_bf16(x[8 * c4 + 6], x[8 * c4 + 7]));
        } else if (live && p.out_bf16) {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + obase + 32 * j);
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4)
            dst[c4] = make_uint4(pack_bf16(x[8 * c4 + 0], x[8 * c4 + 1]), pack_bf16(x[8 * c4 + 2], x[8 * c4 + 3]),
                                 pack_bf16(x[8 * c4 + 4], x[8 * c4 + 5]), pack_bf16(x[8 * c4 + 6], x[8 * c4 + 7]));
        } else if (live) {
          float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out) + obase + 32 * j);
#pragma unroll
          for (int c4 = 0; c4 < 8; ++c4)
            dst[c4] = make_float4(x[4 * c4], x[4 * c4 + 1], x[4 * c4 + 2], x[4 * c4 + 3]);
        }
      }
      if (out_tma && (j & 1)) {                       // uniform over the warpgroup
        // box j/2 is complete: hand it to the TMA engine
        fence_proxy_async_smem();
        epi_sync_c();
        if (leader && go) {
          tma_store_2d(&tmY, io_box(j >> 1), h * p.dv + NV * part + 64 * (j >> 1), t0);
          tma_store_commit();
        }
      }
    }
    if (out_tma && go && leader) tma_store_wait_read();
  }
  if (xchg) {
    if (warp < 2) {
      cluster_wait();
      cluster_arrive();
    }
    cluster_wait();        // the partner has written its statistics: no more remote access here
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// ===========================================================================
// Host side
// ===========================================================================
// Streaming multiprocessors of the current device (queried once per device).
int sm_count() {
  static int cache[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
  if (dev >= 0 && dev < 64 && cache[dev] > 0) return cache[dev];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    n = 148;
  }
  if (dev >= 0 && dev < 64) cache[dev] = n;
  return n;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// 2-D tensor map of 16-bit elements (bf16, or fp16 when `f16`): `rows` rows
// of `inner` elements, row pitch `pitch` elements, box = 64 elements x
// box_rows rows, 128-byte swizzle.
bool make_map(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint64_t pitch,
              uint32_t box_rows, bool f16 = false) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gdim[2] = {inner, rows};
  cuuint64_t gstride[1] = {pitch * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                  const_cast<void*>(base), gdim, gstride, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int NS>
cudaError_t launch_state(const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mw,
                         const CUtensorMap& mv16, const StateParams& sp, cudaStream_t s) {
  const size_t smem = StCfg<NS>::kSmem;
  auto kern = state_kernel<NS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(static_cast<unsigned>(sp.L.nseq) * sp.H * ((sp.dk + 127) / 128) * (sp.dv / NS));
  kern<<<grid, kStThreads, smem, s>>>(mk, mv, mw, mv16, sp);
  return cudaGetLastError();
}

template <int DK, int NV>
cudaError_t launch_out(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                       const CUtensorMap& ms, const CUtensorMap& mg, const CUtensorMap& my,
                       OutParams op, cudaStream_t s) {
  using C = OutCfg<DK, NV>;
  static_assert(C::kSmem <= 232448, "shared memory budget");
  // the dynamic tile order is its own instantiation: the static walk keeps its code
  auto kern = op.dyn ? output_kernel<DK, NV, true> : output_kernel<DK, NV, false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(C::kSmem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = op.parts;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // persistent grid: as many clusters as can be resident at once (one CTA
  // per SM), queried once per device and cluster size
  static int resident[64][3][2] = {};
  int dev = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int& ncl = resident[dev & 63][op.parts][op.dyn ? 1 : 0];
  if (ncl == 0) {
    cfg.gridDim = dim3(static_cast<unsigned>(op.parts), 1, 1);
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) {
      (void)cudaGetLastError();
      n = sm_count() / op.parts;
    }
    ncl = n > 0 ? n : 1;
  }
  op.nclusters = op.ntiles < ncl ? op.ntiles : ncl;
  // rotate the row block every round (an odd stride through the rb row blocks)
  op.shift = (op.nclusters % 2 == 0) ? 1 : 2;
  cfg.gridDim = dim3(static_cast<unsigned>(op.nclusters * op.parts), 1, 1);
  return cudaLaunchKernelEx(&cfg, kern, mq, mk, mv, ms, mg, my, op);
}

// One warp waits on an mbarrier that nothing arrives on, through the bounded
// wait of the kernels above; on expiry that wait raises the time-out error.
__global__ void wait_timeout_selftest_kernel(unsigned* err) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) {
    volatile int* af = &abort_flag;
    (void)mbar_wait(&bar, 0, af, err);
  }
}

template <int DK, int NV>
cudaError_t launch_out_c(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                         const CUtensorMap& ms, const CUtensorMap& mg, const CUtensorMap& my,
                         const OutParams& op, long long slots, cudaStream_t s) {
  using C = OutCfgC<DK, NV>;
  auto kern = output_kernel_c<DK, NV>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(C::kSmem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(slots * op.parts), op.H, 1);
  cfg.blockDim = dim3(kThreadsC, 1, 1);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = op.parts;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, mq, mk, mv, ms, mg, my, op);
}

// fp16 image of v for the P V products of the parallel form (the state pass
// writes it for the chunkwise form).  Exact inside fp16's range; |v| >= 2^16
// (bf16 0x4780 and above, NaN and infinity included) has no fp16 value and
// raises kErrRange.  Eight values per 16-byte access, two accesses in flight
// per thread.
__global__ void __launch_bounds__(256) v16_kernel(const uint4* __restrict__ v,
                                                   uint4* __restrict__ v16, long long n16,
                                                   unsigned* err, int* tile_ctr) {
  if (tile_ctr && blockIdx.x == 0 && threadIdx.x == 0) *tile_ctr = 0;   // for the next kernel
  uint32_t amax = 0;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  auto convert = [&](uint4 w) {
    const uint32_t a[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) amax = __vmaxu2(amax, a[e] & 0x7fff7fffu);
    return make_uint4(bf16x2_to_f16x2(a[0]), bf16x2_to_f16x2(a[1]), bf16x2_to_f16x2(a[2]),
                      bf16x2_to_f16x2(a[3]));
  };
  for (; i + stride < n16; i += 2 * stride) {
    const uint4 w0 = __ldcs(v + i);
    const uint4 w1 = __ldcs(v + i + stride);
    v16[i] = convert(w0);
    v16[i + stride] = convert(w1);
  }
  if (i < n16) v16[i] = convert(__ldcs(v + i));
  const uint32_t big = max(amax & 0xffffu, amax >> 16);
  if (__any_sync(0xffffffffu, big >= 0x4780u) && (threadIdx.x & 31) == 0)
    raise_error(err, kErrRange);
}

cudaError_t launch_output_pass(const void* q, const void* k, const SeqLayout& L,
                               bool has_state_in, void* out, DType out_t, const void* g,
                               DType g_t, const float* gn_w, const float* gn_b, float eps,
                               bool gated, ChunkWorkspace ws, int H, int dk, int dv,
                               const HeadDecay& dec, unsigned* err, cudaStream_t s,
                               bool acc_out, bool anti, StateRead sr, int* tile_ctr);

}  // namespace

cudaError_t launch_wait_timeout_selftest(unsigned* err, cudaStream_t s) {
  wait_timeout_selftest_kernel<<<1, 32, 0, s>>>(err);
  return cudaGetLastError();
}

bool chunkwise_tc_supported(int dk, int dv, int chunk) {
  const bool dk_ok = dk == 64 || dk == 128 || dk == 256;
  const bool dv_ok = dv == 64 || dv == 128 || dv == 256 || dv == 512;
  const bool c_ok = chunk == 64 || chunk == 128 || chunk == 256 || chunk == 512;
  return dk_ok && dv_ok && c_ok;
}

// Chunk length the tensor-core kernels evaluate.  Every chunk length gives the
// same result (the chunkwise form splits the same sum at different points), so
// every requested chunk runs at one length: a single 128-row block, or 256
// tokens when d_v >= 256, where shorter chunks would make the per-chunk state
// (d_k x d_v) cost as much workspace traffic as the chunk's own inputs.  Longer
// chunks only give each 128-row tile more causal key blocks to multiply: for
// d_k = 256, d_v = 512 the forward takes 0.469 ms at 256 against 0.491 at 512
// (and 0.540 at 128); for 128/128 heads 0.251 / 0.285 / 0.317 ms at 128 / 256
// / 512.
int chunkwise_tc_chunk(int chunk, int dv) {
  (void)chunk;
  return dv >= 256 ? 256 : 128;
}

cudaError_t launch_chunkwise_tc(int phases, const void* q, const void* k, const void* v,
                                const SeqLayout& L, const float* state_in, bool has_state_in,
                                float* state_out, void* out, DType out_t, const void* g,
                                DType g_t, const float* gn_w, const float* gn_b, float eps,
                                bool gated, ChunkWorkspace ws, int H, int dk, int dv,
                                const HeadDecay& dec, unsigned* err, cudaStream_t s,
                                bool acc_out, bool anti, StateRead sr) {
  if (!chunkwise_tc_supported(dk, dv, L.chunk)) return cudaErrorNotSupported;
  const uint64_t Ttot = static_cast<uint64_t>(L.Ttot > 0 ? L.Ttot : 1);
  cudaError_t e = cudaSuccess;
  if (phases & 1) {
    // ---- state pass ----
    // d_v columns per CTA: the widest of 256/128/64 whose grid still covers
    // most of the SMs (every CTA walks its sequence serially, so a small
    // batch needs narrower blocks to fill the machine)
    int NS = dv >= 256 ? 256 : dv;
    const long long blocks = static_cast<long long>(L.nseq) * H * ((dk + 127) / 128);
    const int sms = sm_count();
    while (NS > 64 && blocks * (dv / NS) * 5 < static_cast<long long>(sms) * 3) NS /= 2;
    StateParams sp;
    sp.L = L;
    sp.chunk_base = ws.chunk_base;
    sp.order = L.cu ? ws.order : nullptr;
    sp.state_in = state_in;
    sp.state_out = state_out;
    sp.write_v16 = ws.v16 != nullptr ? 1 : 0;
    sp.anti = anti ? 1 : 0;
    sp.H = H;
    sp.dk = dk;
    sp.dv = dv;
    sp.dec = dec;
    sp.err = err;
    CUtensorMap mk_st, mv_st, mw_st, mv16_st;
    const uint64_t wrows = static_cast<uint64_t>(ws.nslots) * H * dk;    // fp16 state slots
    const uint64_t hdv = static_cast<uint64_t>(H) * dv;
    std::memset(&mv16_st, 0, sizeof(mv16_st));
    if (!make_map(&mk_st, k, static_cast<uint64_t>(H) * dk, Ttot, static_cast<uint64_t>(H) * dk, 64) ||
        !make_map(&mv_st, v, hdv, Ttot, hdv, 64) ||
        !make_map(&mw_st, ws.states, dv, wrows, dv, dk < 128 ? dk : 128, true) ||
        (ws.v16 && !make_map(&mv16_st, ws.v16, hdv, Ttot, hdv, 64, true)))
      return cudaErrorInvalidValue;
    switch (NS) {
      case 64: e = launch_state<64>(mk_st, mv_st, mw_st, mv16_st, sp, s); break;
      case 128: e = launch_state<128>(mk_st, mv_st, mw_st, mv16_st, sp, s); break;
      default: e = launch_state<256>(mk_st, mv_st, mw_st, mv16_st, sp, s); break;
    }
  }
  if (e != cudaSuccess || L.Ttot == 0 || !(phases & 2)) return e;
  return launch_output_pass(q, k, L, has_state_in, out, out_t, g, g_t, gn_w, gn_b, eps, gated,
                            ws, H, dk, dv, dec, err, s, acc_out, anti, sr, nullptr);
}

namespace {

// The output pass: every 128-row tile of every chunk, on the persistent
// output kernel (or the compact one for one-block chunks).  The chunk length
// is L.chunk, a multiple of 128 (the parallel form runs the whole sequence as
// one chunk).  Reads q, k, the fp16 copy of v (ws.v16) and, for tiles whose
// chunk carries a state in, the fp16 state slots (ws.states).
cudaError_t launch_output_pass(const void* q, const void* k, const SeqLayout& L,
                               bool has_state_in, void* out, DType out_t, const void* g,
                               DType g_t, const float* gn_w, const float* gn_b, float eps,
                               bool gated, ChunkWorkspace ws, int H, int dk, int dv,
                               const HeadDecay& dec, unsigned* err, cudaStream_t s,
                               bool acc_out, bool anti, StateRead sr, int* tile_ctr) {
  if (L.chunk < kRowsPerTile || L.chunk % kRowsPerTile != 0) return cudaErrorInvalidValue;
  // accumulation: float32 and ungated (the persistent kernel)
  if (acc_out && (out_t != DType::F32 || gated)) return cudaErrorInvalidValue;
  const uint64_t Ttot = static_cast<uint64_t>(L.Ttot > 0 ? L.Ttot : 1);
  const int NV = dv > 256 ? 256 : dv;
  OutParams op;
  op.L = L;
  op.chunk_base = ws.chunk_base;
  op.has_state_in = has_state_in;
  op.out = out;
  op.out_bf16 = out_t == DType::BF16;
  op.g = g;
  op.g_bf16 = g_t == DType::BF16;
  op.gn_w = gn_w;
  op.gn_b = gn_b;
  op.eps = eps;
  op.gated = gated ? 1 : 0;
  op.H = H;
  op.dk = dk;
  op.dv = dv;
  op.rb = L.chunk / kRowsPerTile;
  op.parts = dv / NV;
  op.dec = dec;
  op.err = err;
  op.g_tma = (gated && g_t == DType::BF16) ? 1 : 0;
  op.y_tma = out_t == DType::BF16 ? 1 : 0;
  op.acc_out = acc_out ? 1 : 0;
  op.anti = anti ? 1 : 0;
  op.s_kmajor = sr.transposed ? 1 : 0;
  op.dyn = (tile_ctr != nullptr && !gated) ? 1 : 0;
  op.tile_ctr = tile_ctr;
  op.s_col0 = sr.col0;
  if (ws.v16 == nullptr) return cudaErrorInvalidValue;   // written by the state pass
  // a transposed read: the slots hold [dv rows][stored_dv] (dv <= 256, one part)
  if (sr.transposed && (dv > 256 || sr.col0 < 0 || sr.col0 % 64 != 0 || sr.col0 + dk > sr.stored_dv))
    return cudaErrorInvalidValue;
  const uint64_t hdv = static_cast<uint64_t>(H) * dv;
  CUtensorMap mq, mk, mv, ms, mg, my;
  const bool s_ok = sr.transposed
      ? make_map(&ms, ws.states, sr.stored_dv, static_cast<uint64_t>(ws.nslots) * H * dv,
                 sr.stored_dv, static_cast<uint32_t>(NV), true)
      : make_map(&ms, ws.states, dv, static_cast<uint64_t>(ws.nslots) * H * dk, dv, 64, true);
  if (!make_map(&mq, q, static_cast<uint64_t>(H) * dk, Ttot, static_cast<uint64_t>(H) * dk, 128) ||
      !make_map(&mk, k, static_cast<uint64_t>(H) * dk, Ttot, static_cast<uint64_t>(H) * dk, 128) ||
      !make_map(&mv, ws.v16, hdv, Ttot, hdv, 64, true) || !s_ok)
    return cudaErrorInvalidValue;
  // gate and output tiles: [Ttot rows][H*dv] bf16 (maps only built when used)
  std::memset(&mg, 0, sizeof(mg));
  std::memset(&my, 0, sizeof(my));
  if ((op.g_tma && !make_map(&mg, g, hdv, Ttot, hdv, 128)) ||
      (op.y_tma && !make_map(&my, out, hdv, Ttot, hdv, 128)))
    return cudaErrorInvalidValue;
  const long long ntiles = static_cast<long long>(ws.nslots) * H * op.rb;
  if (ntiles >= (1ll << 31)) return cudaErrorInvalidValue;
  op.ntiles = static_cast<int>(ntiles);
  op.nch = (L.T + L.chunk - 1) / L.chunk;
  op.nclusters = 1;
  op.shift = 1;
  // the compact kernel has neither the anti-causal mode, accumulation nor transposed reads
  if (op.rb == 1 && dk <= 128 && dv <= 256 && !anti && !acc_out && !sr.transposed) {
    // one-block chunks: the compact kernel, two CTAs per SM, d_v in parts of <= 128
    op.parts = dv > 128 ? 2 : 1;
    const int NVc = dv / op.parts;
    if (dk == 64) {
      switch (NVc) {
        case 64: return launch_out_c<64, 64>(mq, mk, mv, ms, mg, my, op, ws.nslots, s);
        default: return launch_out_c<64, 128>(mq, mk, mv, ms, mg, my, op, ws.nslots, s);
      }
    }
    switch (NVc) {
      case 64: return launch_out_c<128, 64>(mq, mk, mv, ms, mg, my, op, ws.nslots, s);
      default: return launch_out_c<128, 128>(mq, mk, mv, ms, mg, my, op, ws.nslots, s);
    }
  }
  if (dk == 64) {
    switch (NV) {
      case 64: return launch_out<64, 64>(mq, mk, mv, ms, mg, my, op, s);
      case 128: return launch_out<64, 128>(mq, mk, mv, ms, mg, my, op, s);
      default: return launch_out<64, 256>(mq, mk, mv, ms, mg, my, op, s);
    }
  }
  if (dk == 128) {
    switch (NV) {
      case 64: return launch_out<128, 64>(mq, mk, mv, ms, mg, my, op, s);
      case 128: return launch_out<128, 128>(mq, mk, mv, ms, mg, my, op, s);
      default: return launch_out<128, 256>(mq, mk, mv, ms, mg, my, op, s);
    }
  }
  switch (NV) {
    case 64: return launch_out<256, 64>(mq, mk, mv, ms, mg, my, op, s);
    case 128: return launch_out<256, 128>(mq, mk, mv, ms, mg, my, op, s);
    default: return launch_out<256, 256>(mq, mk, mv, ms, mg, my, op, s);
  }
}

}  // namespace

cudaError_t launch_to_f16(const void* src, void* dst, long long n, unsigned* err, cudaStream_t s) {
  if (n % 8 != 0) return cudaErrorInvalidValue;
  const long long n16 = n / 8;
  if (n16 == 0) return cudaSuccess;
  const long long want = (n16 + 511) / 512;
  const long long cap = static_cast<long long>(sm_count()) * 8;
  const int blocks = static_cast<int>(want < cap ? want : cap);
  v16_kernel<<<blocks, 256, 0, s>>>(static_cast<const uint4*>(src), static_cast<uint4*>(dst), n16, err,
                                    nullptr);
  return cudaGetLastError();
}

bool parallel_tc_supported(int dk, int dv) {
  return (dk == 64 || dk == 128 || dk == 256) &&
         (dv == 64 || dv == 128 || dv == 256 || dv == 512);
}

size_t parallel_tc_workspace_bytes(int B, int T, int H, int dk, int dv) {
  // the fp16 copy of v, at least B*H*d_k rows of d_v long: the output pass
  // also builds its (never read) state-slot map over this buffer
  const long long rows = static_cast<long long>(B) * (T > dk ? T : dk) * H;
  // then 256 bytes for the tile counter of the dynamic tile order
  return ((static_cast<size_t>(rows) * dv * 2 + 255) & ~static_cast<size_t>(255)) + 256;
}

cudaError_t launch_parallel_tc(const void* q, const void* k, const void* v, void* o, DType o_t,
                               int B, int T, int H, int dk, int dv, const HeadDecay& dec,
                               void* workspace, unsigned* err, cudaStream_t s) {
  if (!parallel_tc_supported(dk, dv) || B < 1 || T < 1) return cudaErrorNotSupported;
  // every (b, h) sequence is one chunk of ceil(T/128)*128 tokens with no
  // incoming state: the chunkwise form then reduces to the parallel form
  // (the intra-chunk term is (Q K^T * D) V over the whole sequence)
  SeqLayout L;
  L.cu = nullptr;
  L.nseq = B;
  L.T = T;
  L.Ttot = B * T;
  L.chunk = (T + kRowsPerTile - 1) / kRowsPerTile * kRowsPerTile;
  L.nslots = B;
  ChunkWorkspace ws;
  ws.chunk_base = nullptr;
  ws.order = nullptr;
  ws.states = workspace;
  ws.v16 = workspace;
  ws.nslots = B;
  const long long n16 = static_cast<long long>(B) * T * H * dv / 8;
  const long long want = (n16 + 511) / 512;
  const long long cap = static_cast<long long>(sm_count()) * 8;
  const int blocks = static_cast<int>(want < cap ? (want > 0 ? want : 1) : cap);
  int* ctr = reinterpret_cast<int*>(static_cast<char*>(workspace) +
                                    parallel_tc_workspace_bytes(B, T, H, dk, dv) - 256);
  v16_kernel<<<blocks, 256, 0, s>>>(static_cast<const uint4*>(v), static_cast<uint4*>(workspace),
                                    n16, err, ctr);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // rows of a sequence cost 1 .. T/128 key blocks: the tiles go out in a dynamic order
  return launch_output_pass(q, k, L, false, o, o_t, nullptr, DType::BF16, nullptr, nullptr, 0.f,
                            false, ws, H, dk, dv, dec, err, s, false, false, StateRead(), ctr);
}

}  // namespace ret

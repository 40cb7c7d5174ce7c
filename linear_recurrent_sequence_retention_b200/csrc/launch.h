// Internal host-side launchers of libretention (not part of the C ABI).
// Arguments are validated by the entry points in api.cu before these run.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "common.cuh"

namespace ret {

enum class DType { F32 = 0, BF16 = 1 };

// Workspace layout of the chunkwise forward:
//   [meta: chunk_base int32[nseq+1], rounded up to 256 B][states][v16]
// states hold the state entering every chunk, one slot per chunk:
//   [slot][H][dk][dv], float32 on the CUDA-core path, fp16 on the tensor-core
//   path (the MMA operand of the cross-chunk read).  v16 (tensor-core path
//   only, at a 256-byte boundary) is the fp16 copy of v, [Ttot][H][dv], that
//   the state pass writes for the output pass's P V products.
struct ChunkWorkspace {
  int32_t* chunk_base;   // device, nseq+1 entries (varlen only; else unused)
  int32_t* order;        // device, nseq entries: sequences longest first (varlen only)
  void* states;          // device
  void* v16;             // device (tensor-core path), else nullptr
  long long nslots;      // slots available
};

size_t chunkwise_meta_bytes(int nseq);

// CUDA-core (fp32 FFMA) kernels.
cudaError_t launch_parallel_simt(const void* q, const void* k, const void* v, DType in_t,
                                 void* o, DType o_t, int B, int T, int H, int dk, int dv,
                                 const HeadDecay& dec, cudaStream_t s);

cudaError_t launch_chunk_prep(const SeqLayout& L, ChunkWorkspace ws, unsigned* err,
                              cudaStream_t s);

// phases: bit 0 = state pass (per-chunk states into the workspace, state_out),
//         bit 1 = output pass (reads the workspace written by a state pass).
cudaError_t launch_chunkwise_simt(int phases, const void* q, const void* k, const void* v,
                                  DType in_t,
                                  const SeqLayout& L, const float* state_in, float* state_out,
                                  void* out, DType out_t, const void* g, DType g_t,
                                  const float* gn_w, const float* gn_b, float eps, bool gated,
                                  ChunkWorkspace ws, int H, int dk, int dv,
                                  const HeadDecay& dec, unsigned* err, cudaStream_t s);

// Workspace of the chunkwise backward: [meta as above][forward states][backward
// states], both [slot][H][dk][dv] float32.
struct ChunkBwdWorkspace {
  int32_t* chunk_base;   // device, nseq+1 entries (varlen only)
  int32_t* order;        // device, nseq entries (varlen only)
  float* fwd_states;     // state entering each chunk
  float* bwd_states;     // gradient state of everything after each chunk
  long long nslots;
};

// CUDA-core backward of the chunkwise form (f32 or bf16 inputs, f32 gradients).
cudaError_t launch_chunkwise_bwd_simt(const void* q, const void* k, const void* v,
                                      const void* d_out, DType in_t, const SeqLayout& L,
                                      const float* state_in, const float* d_state_out, float* dq,
                                      float* dk, float* dv, float* d_state_in,
                                      const ChunkBwdWorkspace& ws, int H, int dk_, int dv_,
                                      const HeadDecay& dec, cudaStream_t s);

// Backward on the tensor-core forward kernels (bf16 inputs, d_k and d_v in
// {64, 128, 256}; with a final-state gradient, every gamma 0 or >= 1e-6): three
// forward retentions with the operand roles exchanged, two of them on the
// sequences read backwards.  `ws`
// holds the chunk offsets and one set of hi/lo states (reused by the three
// passes); `scratch` (chunkwise_bwd_tc_scratch_bytes) the reversed inputs and
// outputs and S0^T.
size_t chunkwise_bwd_tc_scratch_bytes(const SeqLayout& L, int H, int dk, int dv);
cudaError_t launch_chunkwise_bwd_tc(const void* q, const void* k, const void* v,
                                    const void* d_out, const SeqLayout& L, const float* state_in,
                                    const float* d_state_out, float* dq, float* dk, float* dv,
                                    float* d_state_in, ChunkWorkspace ws, void* scratch, int H,
                                    int dk_, int dv_, const HeadDecay& dec, unsigned* err,
                                    cudaStream_t s);

// Rotary position encoding of q and k: [Ttot][H][d], positions counted from
// each sequence's first token; qo/ko may alias q/k.
cudaError_t launch_rope(const void* q, const void* k, DType t, void* qo, void* ko,
                        const SeqLayout& L, int H, int d, double base, cudaStream_t s);

// Inputs of the residual linear attention: qf = phi(q), ks[n] = phi(k[n-w-1]),
// vs[n] = v[n-w-1] (zero before each sequence), phi = softmax over the head dim.
cudaError_t launch_rla_inputs(const void* q, const void* k, const void* v, DType t, void* qf,
                              void* ks, void* vs, const SeqLayout& L, int H, int dk, int dv,
                              int window, cudaStream_t s);

// Tn (1..16) tokens per sequence in one pass over the state.
cudaError_t launch_decode_steps(const void* q, const void* k, const void* v, DType in_t,
                                float* state, void* o, DType o_t, int N, int Tn, int H, int dk,
                                int dv, const HeadDecay& dec, unsigned* err, cudaStream_t s);
// Tn decode steps on the tensor cores (bf16 q, k, v; tf32 MMAs on the float32
// state; d_k in {128, 256}, d_v a multiple of 128 whose operand tiles fit).
bool decode_steps_tc_supported(int Tn, int dk, int dv);
bool decode_steps_tc_preferred(int Tn, int dk, int dv);
cudaError_t launch_decode_steps_tc(const void* q, const void* k, const void* v, float* state,
                                   void* o, DType o_t, int N, int Tn, int H, int dk, int dv,
                                   const HeadDecay& dec, unsigned* err, cudaStream_t s);
cudaError_t launch_decode_step(const void* q, const void* k, const void* v, DType in_t,
                               float* state, void* o, DType o_t, int N, int H, int dk, int dv,
                               const HeadDecay& dec, cudaStream_t s);

cudaError_t launch_norm_gate(const void* o, DType o_t, const void* g, DType g_t,
                             const float* w, const float* b, float eps, void* y, DType y_t,
                             int ntok, int H, int dv, cudaStream_t s);

// Tensor-core (tcgen05) chunkwise forward for bf16 inputs.
bool chunkwise_tc_supported(int dk, int dv, int chunk);

// One bounded wait that is never satisfied (failure-detection self-test).
cudaError_t launch_wait_timeout_selftest(unsigned* err, cudaStream_t s);
int chunkwise_tc_chunk(int chunk, int dv);  // chunk length the kernels evaluate
// The output pass may read the carried state transposed: the slots then hold
// another pass's state [dv rows][stored_dv columns] (fp16) and this pass uses
// its columns col0 .. col0+dk-1 (the backward's dK pass on the dV pass's states).
struct StateRead {
  bool transposed = false;
  int col0 = 0;
  int stored_dv = 0;
};
cudaError_t launch_chunkwise_tc(int phases, const void* q, const void* k, const void* v,
                                const SeqLayout& L, const float* state_in, bool has_state_in,
                                float* state_out,
                                void* out, DType out_t, const void* g, DType g_t,
                                const float* gn_w, const float* gn_b, float eps, bool gated,
                                ChunkWorkspace ws, int H, int dk, int dv,
                                const HeadDecay& dec, unsigned* err, cudaStream_t s,
                                bool acc_out = false, bool anti = false,
                                StateRead sr = StateRead());
// bf16 -> fp16 copy of n elements (n a multiple of 8); |x| >= 2^16 raises kErrRange.
cudaError_t launch_to_f16(const void* src, void* dst, long long n, unsigned* err, cudaStream_t s);

// Parallel form on the tensor cores (bf16 inputs): an fp16 copy of v, then the
// chunkwise output kernel with each sequence as a single chunk.
bool parallel_tc_supported(int dk, int dv);
size_t parallel_tc_workspace_bytes(int B, int T, int H, int dk, int dv);
cudaError_t launch_parallel_tc(const void* q, const void* k, const void* v, void* o, DType o_t,
                               int B, int T, int H, int dk, int dv, const HeadDecay& dec,
                               void* workspace, unsigned* err, cudaStream_t s);

}  // namespace ret

// C ABI of libretention.so (declared in include/retention.h): argument
// validation, per-head decay constants, the per-device error word, and
// dispatch to the kernels.  No entry point allocates device memory: the
// chunkwise forward takes a caller-owned workspace sized by
// retention_chunkwise_workspace_size().
#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include "retention.h"
#include "launch.h"

namespace {

using ret::DType;

// Per-device error word; kernels atomicOr ret::kErr* bits into it instead of
// trapping.  Host code needs the device address, resolved once per device.
__device__ unsigned int g_error_word;

constexpr int kMaxDevices = 64;
std::mutex g_err_mu;
unsigned* g_err_addr[kMaxDevices] = {};

unsigned* error_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_err_mu);
  if (g_err_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_error_word) != cudaSuccess) return nullptr;
    g_err_addr[dev] = static_cast<unsigned*>(p);
  }
  return g_err_addr[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool dtype_ok(ret_dtype t) { return t == RET_F32 || t == RET_BF16; }
DType dt(ret_dtype t) { return t == RET_F32 ? DType::F32 : DType::BF16; }

bool make_decay(const double* gamma, int H, ret::HeadDecay* d) {
  if (gamma == nullptr || H < 1 || H > ret::kMaxHeads) return false;
  std::memset(d, 0, sizeof(*d));
  for (int h = 0; h < H; ++h) {
    double g = gamma[h];
    if (!std::isfinite(g) || g < 0.0 || g > 1.0) return false;
    d->gamma[h] = static_cast<float>(g);
    if (g == 0.0) {
      d->zero_mask |= 1ull << h;
      d->log2g[h] = 0.f;
    } else {
      d->log2g[h] = static_cast<float>(std::log2(g));
    }
  }
  return true;
}

ret_status cuda_status(cudaError_t e) { return e == cudaSuccess ? RET_OK : RET_ERR_CUDA; }

bool fits_int(long long x) { return x >= 0 && x < (1ll << 31); }

size_t round256(size_t b) { return (b + 255) / 256 * 256; }

// Bytes of the tensor-core path's fp16 per-chunk states, and of its fp16 copy
// of v (`width` values per token and head), each rounded to 256 B.
size_t tc_state_bytes(long long slots, int H, int dk, int dv) {
  return round256(static_cast<size_t>(slots) * H * dk * dv * 2);
}
size_t tc_v16_bytes(long long Ttot, int H, int width) {
  return round256(static_cast<size_t>(Ttot) * H * width * 2);
}

struct ChunkPlan {
  ret::SeqLayout L;
  bool tc;
  size_t meta;
  long long slots;
  size_t v16_off;     // tensor-core path: offset of the fp16 copy of v (else 0)
  size_t bytes;
};

// Shared by the size query and the forward call.
ret_status plan_chunkwise(ret_dtype in_dtype, int chunk, int B, int T, int H, int dk, int dv,
                          int nseq, const int32_t* cu, ChunkPlan* p) {
  if (!dtype_ok(in_dtype) || chunk < 1 || H < 1 || H > ret::kMaxHeads || dk < 1 || dv < 1)
    return RET_ERR_INVALID_ARG;
  const bool varlen = nseq > 0;
  if (nseq < 0) return RET_ERR_INVALID_ARG;
  if (varlen) {
    if (B != 1 || T < 0) return RET_ERR_INVALID_ARG;
  } else if (B < 1 || T < 1) {
    return RET_ERR_INVALID_ARG;
  }
  const long long Ttot = varlen ? T : static_cast<long long>(B) * T;
  const int dmax = dk > dv ? dk : dv;
  if (!fits_int(Ttot * H * static_cast<long long>(dmax)) || !fits_int(Ttot + chunk))
    return RET_ERR_INVALID_ARG;
  int ce = chunk;
  if (in_dtype == RET_BF16) {
    if (!ret::chunkwise_tc_supported(dk, dv, chunk)) return RET_ERR_UNSUPPORTED;
    ce = ret::chunkwise_tc_chunk(chunk, dv);
    p->tc = true;
  } else {
    if (dk > 256 || dv > 256) return RET_ERR_UNSUPPORTED;
    p->tc = false;
  }
  p->L.cu = varlen ? cu : nullptr;
  p->L.nseq = varlen ? nseq : B;
  p->L.T = varlen ? 0 : T;
  p->L.Ttot = static_cast<int>(Ttot);
  p->L.chunk = ce;
  p->meta = ret::chunkwise_meta_bytes(p->L.nseq);
  // one slot per chunk; a packed batch has at most ceil(Ttot/ce) + nseq chunks
  p->slots = varlen ? (Ttot + ce - 1) / ce + nseq
                    : static_cast<long long>(B) * ((T + ce - 1) / ce);
  p->L.nslots = p->slots;
  if (p->tc) {
    // fp16 states, then the fp16 copy of v written by the state pass
    p->v16_off = p->meta + tc_state_bytes(p->slots, H, dk, dv);
    p->bytes = p->v16_off + tc_v16_bytes(Ttot, H, dv);
  } else {
    p->v16_off = 0;
    p->bytes = p->meta + static_cast<size_t>(p->slots) * H * dk * dv * sizeof(float);
  }
  return RET_OK;
}

}  // namespace

extern "C" {

int retention_abi_version(void) { return RETENTION_ABI_VERSION; }

// The build passes the SHA-256 of the sources as RET_SOURCE_SHA (a bare hex token).
#ifndef RET_SOURCE_SHA
#define RET_SOURCE_SHA unknown
#endif
#define RET_STR2(x) #x
#define RET_STR(x) RET_STR2(x)
const char* retention_source_sha(void) { return RET_STR(RET_SOURCE_SHA); }

const char* retention_status_string(ret_status s) {
  switch (s) {
    case RET_OK: return "RET_OK";
    case RET_ERR_INVALID_ARG: return "RET_ERR_INVALID_ARG: invalid argument";
    case RET_ERR_UNSUPPORTED: return "RET_ERR_UNSUPPORTED: no kernel for this shape/dtype";
    case RET_ERR_CUDA: return "RET_ERR_CUDA: CUDA call failed";
    case RET_ERR_TIMEOUT: return "RET_ERR_TIMEOUT: a bounded device wait expired";
    case RET_ERR_WORKSPACE: return "RET_ERR_WORKSPACE: workspace missing or too small";
    case RET_ERR_DEVICE_DATA: return "RET_ERR_DEVICE_DATA: inconsistent cu_seqlens";
    case RET_ERR_RANGE:
      return "RET_ERR_RANGE: a value exceeded the fp16 range of the tensor-core operands";
  }
  return "unknown ret_status";
}

size_t retention_parallel_workspace_size(ret_dtype in_dtype, int B, int T, int H, int dk,
                                         int dv) {
  if (in_dtype != RET_BF16 || !ret::parallel_tc_supported(dk, dv) || B < 1 || T < 1 || H < 1)
    return 0;
  const int dmax = dk > dv ? dk : dv;
  const long long tt = static_cast<long long>(B) * (T > dk ? T : dk);
  if (!fits_int(tt * H * dmax)) return 0;
  return ret::parallel_tc_workspace_bytes(B, T, H, dk, dv);
}

ret_status retention_parallel_fwd(const void* q, const void* k, const void* v,
                                  ret_dtype in_dtype, const double* gamma, void* o,
                                  ret_dtype o_dtype, void* workspace, size_t workspace_bytes,
                                  int B, int T, int H, int dk, int dv, ret_stream_t stream) {
  if (!q || !k || !v || !o || !dtype_ok(in_dtype) || !dtype_ok(o_dtype)) return RET_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return RET_ERR_INVALID_ARG;
  if (B < 1 || T < 1 || H < 1 || dk < 1 || dv < 1) return RET_ERR_INVALID_ARG;
  ret::HeadDecay dec;
  if (!make_decay(gamma, H, &dec)) return RET_ERR_INVALID_ARG;
  const int dmax = dk > dv ? dk : dv;
  if (!fits_int(static_cast<long long>(B) * T * H * dmax)) return RET_ERR_INVALID_ARG;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t need = retention_parallel_workspace_size(in_dtype, B, T, H, dk, dv);
  if (need > 0) {
    if (workspace == nullptr || workspace_bytes < need ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
      return RET_ERR_WORKSPACE;
    unsigned* err = error_word();
    if (!err) return RET_ERR_CUDA;
    return cuda_status(ret::launch_parallel_tc(q, k, v, o, dt(o_dtype), B, T, H, dk, dv, dec,
                                               workspace, err, s));
  }
  if (dk > 256 || dv > 256) return RET_ERR_UNSUPPORTED;
  return cuda_status(ret::launch_parallel_simt(q, k, v, dt(in_dtype), o, dt(o_dtype), B, T, H,
                                               dk, dv, dec, s));
}

size_t retention_chunkwise_workspace_size(ret_dtype in_dtype, int chunk, int B, int T, int H,
                                          int dk, int dv, int nseq) {
  ChunkPlan p;
  if (plan_chunkwise(in_dtype, chunk, B, T, H, dk, dv, nseq, nullptr, &p) != RET_OK) return 0;
  return p.bytes;
}

int retention_chunkwise_executed_chunk(ret_dtype in_dtype, int chunk, int dk, int dv) {
  ChunkPlan p;
  if (plan_chunkwise(in_dtype, chunk, 1, chunk, 1, dk, dv, 0, nullptr, &p) != RET_OK) return 0;
  return p.L.chunk;
}

}  // extern "C"

namespace {

// Validated arguments of one chunkwise call (any phase).
struct ChunkCall {
  ChunkPlan p;
  ret::HeadDecay dec;
  const void* g = nullptr;
  DType g_t = DType::F32;
  const float* gw = nullptr;
  const float* gb = nullptr;
  float eps = 0.f;
  ret::ChunkWorkspace ws;
  unsigned* err = nullptr;
};

constexpr int kPhaseStates = 1, kPhaseOutputs = 2;

ret_status prepare_chunk_call(int phases, const void* q, const void* k, const void* v,
                              ret_dtype in_dtype, const double* gamma, int chunk,
                              const int32_t* cu_seqlens, int nseq, const float* state_in,
                              const float* state_out, const void* out, ret_dtype out_dtype,
                              const ret_norm_gate* ng, const void* workspace,
                              size_t workspace_bytes, int B, int T, int H, int dk, int dv,
                              ChunkCall* c) {
  const bool varlen = cu_seqlens != nullptr;
  if (varlen != (nseq > 0)) return RET_ERR_INVALID_ARG;
  ret_status st = plan_chunkwise(in_dtype, chunk, B, T, H, dk, dv, varlen ? nseq : 0,
                                 cu_seqlens, &c->p);
  if (st != RET_OK) return st;
  const bool has_tokens = c->p.L.Ttot > 0;
  if (has_tokens && (!k || !v)) return RET_ERR_INVALID_ARG;
  if ((phases & kPhaseOutputs) && has_tokens && (!q || !out)) return RET_ERR_INVALID_ARG;
  if ((phases & kPhaseOutputs) && !dtype_ok(out_dtype)) return RET_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, out, state_in, state_out, cu_seqlens};
  for (const void* ptr : ptrs)
    if (ptr && !aligned16(ptr)) return RET_ERR_INVALID_ARG;
  if (!make_decay(gamma, H, &c->dec)) return RET_ERR_INVALID_ARG;
  if (ng && (phases & kPhaseOutputs)) {
    if (!ng->g || !dtype_ok(ng->g_dtype) || !aligned16(ng->g)) return RET_ERR_INVALID_ARG;
    if (!std::isfinite(ng->eps) || ng->eps < 0.f) return RET_ERR_INVALID_ARG;
    c->g = ng->g;
    c->g_t = dt(ng->g_dtype);
    c->gw = ng->weight;
    c->gb = ng->bias;
    c->eps = ng->eps;
  }
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 ||
      workspace_bytes < c->p.bytes)
    return RET_ERR_WORKSPACE;
  c->ws.chunk_base = static_cast<int32_t*>(const_cast<void*>(workspace));
  c->ws.order = c->ws.chunk_base + c->p.L.nseq + 1;
  c->ws.states = static_cast<char*>(const_cast<void*>(workspace)) + c->p.meta;
  c->ws.v16 = c->p.v16_off ? static_cast<char*>(const_cast<void*>(workspace)) + c->p.v16_off
                           : nullptr;
  c->ws.nslots = c->p.slots;
  c->err = error_word();
  if (!c->err) return RET_ERR_CUDA;
  return RET_OK;
}

ret_status run_chunk_call(int phases, const ChunkCall& c, const void* q, const void* k,
                          const void* v, ret_dtype in_dtype, const float* state_in,
                          bool has_state_in, float* state_out, void* out, ret_dtype out_dtype,
                          bool gated, int H, int dk, int dv, cudaStream_t s) {
  cudaError_t e = cudaSuccess;
  if (phases & kPhaseStates) {
    e = ret::launch_chunk_prep(c.p.L, c.ws, c.err, s);
    if (e != cudaSuccess) return RET_ERR_CUDA;
  }
  if (c.p.tc)
    e = ret::launch_chunkwise_tc(phases, q, k, v, c.p.L, state_in, has_state_in, state_out, out,
                                 dt(out_dtype), c.g, c.g_t, c.gw, c.gb, c.eps, gated, c.ws, H, dk,
                                 dv, c.dec, c.err, s);
  else
    e = ret::launch_chunkwise_simt(phases, q, k, v, dt(in_dtype), c.p.L, state_in, state_out,
                                   out, dt(out_dtype), c.g, c.g_t, c.gw, c.gb, c.eps, gated, c.ws,
                                   H, dk, dv, c.dec, c.err, s);
  return cuda_status(e);
}

}  // namespace

extern "C" {

ret_status retention_chunkwise_fwd(const void* q, const void* k, const void* v,
                                   ret_dtype in_dtype, const double* gamma, int chunk,
                                   const int32_t* cu_seqlens, int nseq,
                                   const float* state_in, float* state_out,
                                   void* out, ret_dtype out_dtype, const ret_norm_gate* ng,
                                   void* workspace, size_t workspace_bytes,
                                   int B, int T, int H, int dk, int dv,
                                   ret_stream_t stream) {
  const int ph = kPhaseStates | kPhaseOutputs;
  ChunkCall c;
  ret_status st = prepare_chunk_call(ph, q, k, v, in_dtype, gamma, chunk, cu_seqlens, nseq,
                                     state_in, state_out, out, out_dtype, ng, workspace,
                                     workspace_bytes, B, T, H, dk, dv, &c);
  if (st != RET_OK) return st;
  return run_chunk_call(ph, c, q, k, v, in_dtype, state_in, state_in != nullptr, state_out, out,
                        out_dtype, ng != nullptr, H, dk, dv,
                        reinterpret_cast<cudaStream_t>(stream));
}

size_t retention_chunkwise_fwd_rope_workspace_size(int chunk, int B, int T, int H, int dk,
                                                    int dv, int nseq) {
  ChunkPlan p;
  if (plan_chunkwise(RET_BF16, chunk, B, T, H, dk, dv, nseq, nullptr, &p) != RET_OK) return 0;
  const size_t rows = static_cast<size_t>(p.L.Ttot) * H * dk * 2;
  return round256(p.bytes) + 2 * round256(rows);
}

ret_status retention_chunkwise_fwd_rope(const void* q, const void* k, const void* v,
                                        ret_dtype in_dtype, const double* gamma, int chunk,
                                        const int32_t* cu_seqlens, int nseq,
                                        const float* state_in, float* state_out, void* out,
                                        ret_dtype out_dtype, const ret_norm_gate* ng,
                                        double rope_base, void* workspace,
                                        size_t workspace_bytes, int B, int T, int H, int dk,
                                        int dv, ret_stream_t stream) {
  if (in_dtype != RET_BF16) return RET_ERR_UNSUPPORTED;
  if (!std::isfinite(rope_base) || rope_base <= 1.0 || (dk & 1)) return RET_ERR_INVALID_ARG;
  const int ph = kPhaseStates | kPhaseOutputs;
  const size_t need = retention_chunkwise_fwd_rope_workspace_size(chunk, B, T, H, dk, dv,
                                                                  cu_seqlens ? nseq : 0);
  ChunkCall c;
  // the chunkwise part of the workspace comes first; the rotated q and k follow it
  ret_status st = prepare_chunk_call(ph, q, k, v, in_dtype, gamma, chunk, cu_seqlens, nseq,
                                     state_in, state_out, out, out_dtype, ng, workspace,
                                     workspace_bytes, B, T, H, dk, dv, &c);
  if (st != RET_OK) return st;
  if (workspace_bytes < need) return RET_ERR_WORKSPACE;
  char* rot = static_cast<char*>(workspace) + round256(c.p.bytes);
  void* q_rot = rot;
  void* k_rot = rot + round256(static_cast<size_t>(c.p.L.Ttot) * H * dk * 2);
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = ret::launch_chunk_prep(c.p.L, c.ws, c.err, s);
  // one streaming pass rotates q and k into the workspace; the chunkwise
  // passes then read the rotated copies (faster on this GPU than rotating k
  // inside the state pass, whose converter warps set that pass's pace)
  if (e == cudaSuccess)
    e = ret::launch_rope(q, k, DType::BF16, q_rot, k_rot, c.p.L, H, dk, rope_base, s);
  if (e == cudaSuccess)
    e = ret::launch_chunkwise_tc(ph, q_rot, k_rot, v, c.p.L, state_in, state_in != nullptr,
                                 state_out, out, dt(out_dtype), c.g, c.g_t, c.gw, c.gb, c.eps,
                                 ng != nullptr, c.ws, H, dk, dv, c.dec, c.err, s);
  return cuda_status(e);
}

ret_status retention_chunkwise_states(const void* k, const void* v, ret_dtype in_dtype,
                                      const double* gamma, int chunk,
                                      const int32_t* cu_seqlens, int nseq,
                                      const float* state_in, float* state_out,
                                      void* workspace, size_t workspace_bytes,
                                      int B, int T, int H, int dk, int dv,
                                      ret_stream_t stream) {
  const int ph = kPhaseStates;
  ChunkCall c;
  ret_status st = prepare_chunk_call(ph, nullptr, k, v, in_dtype, gamma, chunk, cu_seqlens,
                                     nseq, state_in, state_out, nullptr, RET_F32, nullptr,
                                     workspace, workspace_bytes, B, T, H, dk, dv, &c);
  if (st != RET_OK) return st;
  return run_chunk_call(ph, c, nullptr, k, v, in_dtype, state_in, state_in != nullptr,
                        state_out, nullptr, RET_F32, false, H, dk, dv,
                        reinterpret_cast<cudaStream_t>(stream));
}

ret_status retention_chunkwise_outputs(const void* q, const void* k, const void* v,
                                       ret_dtype in_dtype, const double* gamma, int chunk,
                                       const int32_t* cu_seqlens, int nseq, int has_state_in,
                                       void* out, ret_dtype out_dtype, const ret_norm_gate* ng,
                                       const void* workspace, size_t workspace_bytes,
                                       int B, int T, int H, int dk, int dv,
                                       ret_stream_t stream) {
  const int ph = kPhaseOutputs;
  ChunkCall c;
  ret_status st = prepare_chunk_call(ph, q, k, v, in_dtype, gamma, chunk, cu_seqlens, nseq,
                                     nullptr, nullptr, out, out_dtype, ng, workspace,
                                     workspace_bytes, B, T, H, dk, dv, &c);
  if (st != RET_OK) return st;
  return run_chunk_call(ph, c, q, k, v, in_dtype, nullptr, has_state_in != 0, nullptr, out,
                        out_dtype, ng != nullptr, H, dk, dv,
                        reinterpret_cast<cudaStream_t>(stream));
}

ret_status retention_recurrent_step(const void* q, const void* k, const void* v,
                                    ret_dtype in_dtype, const double* gamma, float* state,
                                    void* o, ret_dtype o_dtype, int N, int H, int dk, int dv,
                                    ret_stream_t stream) {
  if (!q || !k || !v || !state || !o || !dtype_ok(in_dtype) || !dtype_ok(o_dtype))
    return RET_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(state) || !aligned16(o))
    return RET_ERR_INVALID_ARG;
  if (N < 1 || H < 1 || dk < 1 || dv < 1) return RET_ERR_INVALID_ARG;
  ret::HeadDecay dec;
  if (!make_decay(gamma, H, &dec)) return RET_ERR_INVALID_ARG;
  if (dk > 1024 || dv > 4096) return RET_ERR_UNSUPPORTED;
  if (static_cast<long long>(N) * H > 65535ll * 65535ll || N > 65535 || H > 65535)
    return RET_ERR_UNSUPPORTED;
  return cuda_status(ret::launch_decode_step(q, k, v, dt(in_dtype), state, o, dt(o_dtype), N, H,
                                             dk, dv, dec, reinterpret_cast<cudaStream_t>(stream)));
}

ret_status retention_recurrent_steps(const void* q, const void* k, const void* v,
                                     ret_dtype in_dtype, const double* gamma, float* state,
                                     void* o, ret_dtype o_dtype, int N, int Tn, int H, int dk,
                                     int dv, ret_stream_t stream) {
  if (!q || !k || !v || !state || !o || !dtype_ok(in_dtype) || !dtype_ok(o_dtype))
    return RET_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(state) || !aligned16(o))
    return RET_ERR_INVALID_ARG;
  if (N < 1 || Tn < 1 || H < 1 || dk < 1 || dv < 1) return RET_ERR_INVALID_ARG;
  ret::HeadDecay dec;
  if (!make_decay(gamma, H, &dec)) return RET_ERR_INVALID_ARG;
  if (Tn > 16 || dk > 512 || dv > 4096 || dk % 4 != 0 || dv % 4 != 0) return RET_ERR_UNSUPPORTED;
  if (N > 65535 || H > 65535) return RET_ERR_UNSUPPORTED;
  return cuda_status(ret::launch_decode_steps(q, k, v, dt(in_dtype), state, o, dt(o_dtype), N, Tn,
                                              H, dk, dv, dec, error_word(),
                                              reinterpret_cast<cudaStream_t>(stream)));
}

ret_status msr_norm_gate(const void* o, ret_dtype o_dtype, const ret_norm_gate* ng, void* y,
                         ret_dtype y_dtype, int ntok, int H, int dv, ret_stream_t stream) {
  if (!o || !ng || !ng->g || !y || !dtype_ok(o_dtype) || !dtype_ok(y_dtype) ||
      !dtype_ok(ng->g_dtype))
    return RET_ERR_INVALID_ARG;
  if (!aligned16(o) || !aligned16(ng->g) || !aligned16(y)) return RET_ERR_INVALID_ARG;
  if (ntok < 1 || H < 1 || dv < 1) return RET_ERR_INVALID_ARG;
  if (!std::isfinite(ng->eps) || ng->eps < 0.f) return RET_ERR_INVALID_ARG;
  if (!fits_int(static_cast<long long>(ntok) * H * dv)) return RET_ERR_INVALID_ARG;
  if (dv > 1024) return RET_ERR_UNSUPPORTED;
  return cuda_status(ret::launch_norm_gate(o, dt(o_dtype), ng->g, dt(ng->g_dtype), ng->weight,
                                           ng->bias, ng->eps, y, dt(y_dtype), ntok, H, dv,
                                           reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"

namespace {

struct BwdPlan {
  ret::SeqLayout L;     // CUDA-core path: the caller's chunk
  size_t meta;
  long long slots;
  size_t state_bytes;   // one set of per-chunk float32 states
  size_t bytes;         // CUDA-core path
  bool simt_ok;         // the CUDA-core path is possible (heads up to 256)
  bool tc_ok;           // the tensor-core path is possible (bf16, d_k 64/128/256, d_v 64..512)
  ret::SeqLayout Ltc;   // tensor-core path: the executed chunk
  size_t tc_state;      // one set of fp16 states at that chunk
  size_t tc_states;     // + the fp16 copy of the value operand (the wider of d_k, d_v)
  size_t tc_bytes;      // tensor-core path: meta + states + scratch
};

bool tc_head(int d) { return d == 64 || d == 128 || d == 256; }

// Shared by the backward's size query and call.  The CUDA-core path (float32
// arithmetic, f32 or bf16 inputs, heads up to 256) takes any arguments; bf16
// inputs with d_k in {64, 128, 256}, d_v in {64, 128, 256, 512} and a chunk of
// 64..512 may also run on the tensor-core forward kernels (see
// launch_chunkwise_bwd_tc; d_v = 512 only there), and the workspace is sized
// for whichever possible path needs more.
ret_status plan_chunkwise_bwd(ret_dtype in_dtype, int chunk, int B, int T, int H, int dk, int dv,
                              int nseq, const int32_t* cu, BwdPlan* p) {
  if (!dtype_ok(in_dtype) || chunk < 1 || H < 1 || H > ret::kMaxHeads || dk < 1 || dv < 1 ||
      nseq < 0)
    return RET_ERR_INVALID_ARG;
  const bool varlen = nseq > 0;
  if (varlen) {
    if (B != 1 || T < 0) return RET_ERR_INVALID_ARG;
  } else if (B < 1 || T < 1) {
    return RET_ERR_INVALID_ARG;
  }
  const long long Ttot = varlen ? T : static_cast<long long>(B) * T;
  const int dmax = dk > dv ? dk : dv;
  if (!fits_int(Ttot * H * static_cast<long long>(dmax)) || !fits_int(Ttot + chunk))
    return RET_ERR_INVALID_ARG;
  const bool tc_shape = in_dtype == RET_BF16 && tc_head(dk) && (tc_head(dv) || dv == 512);
  p->simt_ok = dk <= 256 && dv <= 256;
  if (!p->simt_ok && !tc_shape) return RET_ERR_UNSUPPORTED;
  p->L.cu = varlen ? cu : nullptr;
  p->L.nseq = varlen ? nseq : B;
  p->L.T = varlen ? 0 : T;
  p->L.Ttot = static_cast<int>(Ttot);
  p->L.chunk = chunk;
  p->meta = ret::chunkwise_meta_bytes(p->L.nseq);
  p->slots = varlen ? (Ttot + chunk - 1) / chunk + nseq
                    : static_cast<long long>(B) * ((T + chunk - 1) / chunk);
  p->L.nslots = p->slots;
  p->state_bytes = static_cast<size_t>(p->slots) * H * dk * dv * sizeof(float);
  p->bytes = p->meta + 2 * p->state_bytes;
  // the d_v = 512 passes that contract over d_v run on 256-wide halves
  const int dvq = dv > 256 ? dv / 2 : dv;
  p->tc_ok = tc_shape && ret::chunkwise_tc_supported(dk, dv, chunk) &&
             ret::chunkwise_tc_supported(dvq, dk, chunk);
  if (!p->simt_ok && !p->tc_ok) return RET_ERR_UNSUPPORTED;
  p->tc_bytes = 0;
  if (p->tc_ok) {
    // one executed chunk for the three passes (d_k and d_v exchange roles)
    const int ce = ret::chunkwise_tc_chunk(chunk, dk > dv ? dk : dv);
    p->Ltc = p->L;
    p->Ltc.chunk = ce;
    p->Ltc.nslots = varlen ? (Ttot + ce - 1) / ce + nseq
                           : static_cast<long long>(B) * ((T + ce - 1) / ce);
    p->tc_state = tc_state_bytes(p->Ltc.nslots, H, dk, dv);
    p->tc_states = p->tc_state + tc_v16_bytes(Ttot, H, dk > dv ? dk : dv);
    p->tc_bytes = p->meta + p->tc_states + ret::chunkwise_bwd_tc_scratch_bytes(p->Ltc, H, dk, dv);
  }
  return RET_OK;
}

}  // namespace

extern "C" {

size_t retention_chunkwise_bwd_workspace_size(ret_dtype in_dtype, int chunk, int B, int T,
                                              int H, int dk, int dv, int nseq) {
  BwdPlan p;
  if (plan_chunkwise_bwd(in_dtype, chunk, B, T, H, dk, dv, nseq, nullptr, &p) != RET_OK) return 0;
  const size_t a = p.simt_ok ? p.bytes : 0, b = p.tc_ok ? p.tc_bytes : 0;
  return a > b ? a : b;
}

ret_status retention_chunkwise_bwd(const void* q, const void* k, const void* v, const void* d_out,
                                   ret_dtype in_dtype, const double* gamma, int chunk,
                                   const int32_t* cu_seqlens, int nseq, const float* state_in,
                                   const float* d_state_out, float* dq, float* dk, float* dv,
                                   float* d_state_in, void* workspace, size_t workspace_bytes,
                                   int B, int T, int H, int dk_, int dv_, ret_stream_t stream) {
  const bool varlen = cu_seqlens != nullptr;
  if (varlen != (nseq > 0)) return RET_ERR_INVALID_ARG;
  BwdPlan p;
  ret_status st = plan_chunkwise_bwd(in_dtype, chunk, B, T, H, dk_, dv_, varlen ? nseq : 0,
                                     cu_seqlens, &p);
  if (st != RET_OK) return st;
  if (p.L.Ttot > 0 && (!q || !k || !v || !d_out || !dq || !dk || !dv)) return RET_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, d_out, dq, dk, dv, state_in, d_state_out, d_state_in, cu_seqlens};
  for (const void* ptr : ptrs)
    if (ptr && !aligned16(ptr)) return RET_ERR_INVALID_ARG;
  ret::HeadDecay dec;
  if (!make_decay(gamma, H, &dec)) return RET_ERR_INVALID_ARG;
  const bool use_tc = p.tc_ok;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 ||
      workspace_bytes < (use_tc ? p.tc_bytes : p.bytes))
    return RET_ERR_WORKSPACE;
  unsigned* err = error_word();
  if (!err) return RET_ERR_CUDA;
  char* base = static_cast<char*>(workspace);
  if (use_tc) {
    ret::ChunkWorkspace tw;
    tw.chunk_base = reinterpret_cast<int32_t*>(base);
    tw.order = tw.chunk_base + p.Ltc.nseq + 1;
    tw.states = base + p.meta;
    tw.v16 = base + p.meta + p.tc_state;
    tw.nslots = p.Ltc.nslots;
    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = ret::launch_chunk_prep(p.Ltc, tw, err, s);
    if (e == cudaSuccess)
      e = ret::launch_chunkwise_bwd_tc(q, k, v, d_out, p.Ltc, state_in, d_state_out, dq, dk, dv,
                                       d_state_in, tw, base + p.meta + p.tc_states, H, dk_, dv_,
                                       dec, err, s);
    return cuda_status(e);
  }
  ret::ChunkWorkspace fw;
  fw.chunk_base = reinterpret_cast<int32_t*>(base);
  fw.order = fw.chunk_base + p.L.nseq + 1;
  fw.states = base + p.meta;
  fw.v16 = nullptr;
  fw.nslots = p.slots;
  ret::ChunkBwdWorkspace ws;
  ws.chunk_base = fw.chunk_base;
  ws.order = fw.order;
  ws.fwd_states = reinterpret_cast<float*>(base + p.meta);
  ws.bwd_states = reinterpret_cast<float*>(base + p.meta + p.state_bytes);
  ws.nslots = p.slots;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = ret::launch_chunk_prep(p.L, fw, err, s);
  if (e == cudaSuccess)
    e = ret::launch_chunkwise_bwd_simt(q, k, v, d_out, dt(in_dtype), p.L, state_in, d_state_out,
                                       dq, dk, dv, d_state_in, ws, H, dk_, dv_, dec, s);
  return cuda_status(e);
}

ret_status retention_rope(const void* q, const void* k, ret_dtype dtype, void* q_out, void* k_out,
                          double base, const int32_t* cu_seqlens, int nseq, int B, int T, int H,
                          int d, ret_stream_t stream) {
  if (!dtype_ok(dtype) || H < 1 || d < 2 || (d & 1) || d > 65536 || nseq < 0 ||
      !std::isfinite(base) || base <= 1.0)
    return RET_ERR_INVALID_ARG;
  const bool varlen = cu_seqlens != nullptr;
  if (varlen != (nseq > 0)) return RET_ERR_INVALID_ARG;
  if (varlen ? (B != 1 || T < 0) : (B < 1 || T < 1)) return RET_ERR_INVALID_ARG;
  const long long Ttot = varlen ? T : static_cast<long long>(B) * T;
  if (!fits_int(Ttot * H * static_cast<long long>(d))) return RET_ERR_INVALID_ARG;
  if (Ttot > 0 && (!q || !k || !q_out || !k_out)) return RET_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, q_out, k_out, cu_seqlens};
  for (const void* ptr : ptrs)
    if (ptr && !aligned16(ptr)) return RET_ERR_INVALID_ARG;
  ret::SeqLayout L;
  L.cu = varlen ? cu_seqlens : nullptr;
  L.nseq = varlen ? nseq : B;
  L.T = varlen ? 0 : T;
  L.Ttot = static_cast<int>(Ttot);
  L.chunk = 1;
  L.nslots = 0;
  return cuda_status(ret::launch_rope(q, k, dt(dtype), q_out, k_out, L, H, d, base,
                                      reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"

namespace {

// The retention inside RLA runs with 256-token chunks on either path (every
// chunk length gives the same result); the mapped inputs follow its workspace.
constexpr int kRlaChunk = 256;

struct RlaPlan {
  ChunkPlan cp;
  size_t ws_bytes;    // chunk workspace, rounded to 256 B
  size_t bytes;       // + phi(q), shifted phi(k) and v
};

ret_status plan_rla(ret_dtype in_dtype, int B, int T, int H, int dk, int dv, int nseq,
                    const int32_t* cu, RlaPlan* r) {
  ret_status st = plan_chunkwise(in_dtype, kRlaChunk, B, T, H, dk, dv, nseq, cu, &r->cp);
  if (st != RET_OK) return st;
  auto r256 = [](size_t b) { return (b + 255) / 256 * 256; };
  const size_t el = in_dtype == RET_F32 ? 4 : 2;
  const size_t rows = static_cast<size_t>(r->cp.L.Ttot) * H;
  r->ws_bytes = r256(r->cp.bytes);
  r->bytes = r->ws_bytes + 2 * r256(rows * dk * el) + r256(rows * dv * el);
  return RET_OK;
}

}  // namespace

extern "C" {

size_t retention_rla_workspace_size(ret_dtype in_dtype, int B, int T, int H, int dk, int dv,
                                    int nseq) {
  RlaPlan r;
  if (nseq < 0 || plan_rla(in_dtype, B, T, H, dk, dv, nseq, nullptr, &r) != RET_OK) return 0;
  return r.bytes;
}

ret_status retention_rla_fwd(const void* q, const void* k, const void* v, ret_dtype in_dtype,
                             int window, const int32_t* cu_seqlens, int nseq, void* o,
                             ret_dtype o_dtype, void* workspace, size_t workspace_bytes, int B,
                             int T, int H, int dk, int dv, ret_stream_t stream) {
  const bool varlen = cu_seqlens != nullptr;
  if (varlen != (nseq > 0) || window < 0 || !dtype_ok(o_dtype)) return RET_ERR_INVALID_ARG;
  RlaPlan r;
  ret_status st = plan_rla(in_dtype, B, T, H, dk, dv, varlen ? nseq : 0, cu_seqlens, &r);
  if (st != RET_OK) return st;
  if (r.cp.L.Ttot > 0 && (!q || !k || !v || !o)) return RET_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, o, cu_seqlens};
  for (const void* ptr : ptrs)
    if (ptr && !aligned16(ptr)) return RET_ERR_INVALID_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 ||
      workspace_bytes < r.bytes)
    return RET_ERR_WORKSPACE;
  std::vector<double> ones(H, 1.0);
  ret::HeadDecay dec;
  if (!make_decay(ones.data(), H, &dec)) return RET_ERR_INVALID_ARG;
  unsigned* err = error_word();
  if (!err) return RET_ERR_CUDA;
  char* base = static_cast<char*>(workspace);
  ret::ChunkWorkspace ws;
  ws.chunk_base = reinterpret_cast<int32_t*>(base);
  ws.order = ws.chunk_base + r.cp.L.nseq + 1;
  ws.states = base + r.cp.meta;
  ws.v16 = r.cp.v16_off ? base + r.cp.v16_off : nullptr;
  ws.nslots = r.cp.slots;
  auto r256 = [](size_t b) { return (b + 255) / 256 * 256; };
  const size_t el = in_dtype == RET_F32 ? 4 : 2;
  const size_t rows = static_cast<size_t>(r.cp.L.Ttot) * H;
  char* qf = base + r.ws_bytes;
  char* ks = qf + r256(rows * dk * el);
  char* vs = ks + r256(rows * dk * el);
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = ret::launch_chunk_prep(r.cp.L, ws, err, s);
  if (e == cudaSuccess)
    e = ret::launch_rla_inputs(q, k, v, dt(in_dtype), qf, ks, vs, r.cp.L, H, dk, dv, window, s);
  if (e == cudaSuccess) {
    if (r.cp.tc)
      e = ret::launch_chunkwise_tc(3, qf, ks, vs, r.cp.L, nullptr, false, nullptr, o, dt(o_dtype),
                                   nullptr, DType::F32, nullptr, nullptr, 0.f, false, ws, H, dk,
                                   dv, dec, err, s);
    else
      e = ret::launch_chunkwise_simt(3, qf, ks, vs, dt(in_dtype), r.cp.L, nullptr, nullptr, o,
                                     dt(o_dtype), nullptr, DType::F32, nullptr, nullptr, 0.f,
                                     false, ws, H, dk, dv, dec, err, s);
  }
  return cuda_status(e);
}

ret_status retention_selftest_wait_timeout(ret_stream_t stream) {
  unsigned* err = error_word();
  if (!err) return RET_ERR_CUDA;
  return cuda_status(ret::launch_wait_timeout_selftest(err, reinterpret_cast<cudaStream_t>(stream)));
}

ret_status retention_check_device_error(ret_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return RET_ERR_CUDA;
  unsigned* err = error_word();
  if (!err) return RET_ERR_CUDA;
  unsigned word = 0;
  if (cudaMemcpy(&word, err, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
    return RET_ERR_CUDA;
  if (word != 0) {
    const unsigned zero = 0;
    if (cudaMemcpy(err, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
      return RET_ERR_CUDA;
  }
  if (word & ret::kErrTimeout) return RET_ERR_TIMEOUT;
  if (word & ret::kErrDeviceData) return RET_ERR_DEVICE_DATA;
  if (word & ret::kErrRange) return RET_ERR_RANGE;
  return RET_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Chunkwise forward that allocates nothing: its scratch is a file-scope
// device array of RETENTION_STATIC_WORKSPACE_BYTES, present on every device
// that loads this library for as long as the library stays loaded.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kStaticWorkspaceBytes = RETENTION_STATIC_WORKSPACE_BYTES;
static __device__ __align__(256) unsigned char g_static_workspace[kStaticWorkspaceBytes];

std::mutex g_static_mu;
void* g_static_addr[kMaxDevices] = {};

// The host-side name g_static_workspace is only a stand-in for the device
// array: its device address is resolved here, once per device, with that
// device current, and cached for later calls.
void* static_workspace() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_static_mu);
  if (g_static_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_workspace) != cudaSuccess || p == nullptr)
      return nullptr;
    g_static_addr[dev] = p;
  }
  return g_static_addr[dev];
}

}  // namespace

extern "C" {

ret_status retention_chunkwise_fwd_static_ws(const void* q, const void* k, const void* v,
                                             ret_dtype in_dtype, const double* gamma, int chunk,
                                             const int32_t* cu_seqlens, int nseq,
                                             const float* state_in, float* state_out,
                                             void* out, ret_dtype out_dtype,
                                             const ret_norm_gate* ng,
                                             int B, int T, int H, int dk, int dv,
                                             ret_stream_t stream) {
  const size_t need = retention_chunkwise_workspace_size(in_dtype, chunk, B, T, H, dk, dv,
                                                         cu_seqlens ? nseq : 0);
  if (need == 0)   // invalid or unsupported: let the regular validation name the reason
    return retention_chunkwise_fwd(q, k, v, in_dtype, gamma, chunk, cu_seqlens, nseq, state_in,
                                   state_out, out, out_dtype, ng, nullptr, 0, B, T, H, dk, dv,
                                   stream);
  if (need > kStaticWorkspaceBytes) return RET_ERR_WORKSPACE;
  void* ws = static_workspace();
  if (ws == nullptr) return RET_ERR_CUDA;
  return retention_chunkwise_fwd(q, k, v, in_dtype, gamma, chunk, cu_seqlens, nseq, state_in,
                                 state_out, out, out_dtype, ng, ws, kStaticWorkspaceBytes, B, T,
                                 H, dk, dv, stream);
}

}  // extern "C"

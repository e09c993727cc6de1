// Internal declarations shared by the libkda.so translation units.
// Nothing here is part of the public C ABI (include/kda.h).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "kda.h"

namespace kda {

// Bits of the per-device status word (device-side error reporting).
enum : unsigned int {
  STATUS_GATE_RANGE = 1u << 0,   // g outside [-5, 0] or beta outside [0, 1]
  STATUS_TIMEOUT = 1u << 1,      // a bounded wait gave up
  STATUS_BAD_SEQLENS = 1u << 2,  // cu_seqlens inconsistent with total_tokens
};

constexpr int kChunk = KDA_CHUNK;
constexpr float kGateLower = -5.0f;

// Device code reports errors by OR-ing STATUS_* bits into the per-device
// status word whose address the host passes in every parameter block
// (`status`).  Kernels never trap.
__device__ __forceinline__ void set_status(unsigned int *status, unsigned int bits) {
  if (status) atomicOr(status, bits);
}

// Parameters of the chunked prefill kernels (plain pointers, resolved sizes).
struct PrefillParams {
  const void *q, *k, *v;
  const float *g, *beta;
  const __nv_bfloat16 *g_logits;  // when set (g NULL): log(alpha) = -5 sigmoid(logit)
  const int32_t *cu_seqlens;
  const int32_t *order;          // work order over requests (longest first) or NULL
  const float *initial_state;    // NULL = zeros
  void *o;                       // NULL = not written (local-state mode)
  float *final_state;            // NULL = not written
  const int32_t *cu_snapshots;
  float *snapshots;
  int n_req, total_tokens, H, dk, dv;
  int snapshot_stride;
  int n_slices;                  // column slices per (request, head)
  int validate;
  unsigned int *status;
  // Limit of every bounded wait inside the tensor-core kernel, in ns (0: 2 s).
  // Only tests shorten it, to make a wait run out on purpose.
  unsigned long long wait_ns;
  // local-state mode: columns [0, dv) of the augmented state are S_loc (V,
  // zero start), columns [dv, dv + dk) are M (zero V, identity start).
  int local_mode;
  float *s_loc;                  // [n_seg, H, dk, dv]
  float *m;                      // [n_seg, H, dk, dk]
};

struct DecodeParams {
  const void *q, *k, *v;
  const float *g, *beta;
  float *state;
  const int32_t *slot;
  void *o;
  int n, H, dk, dv, n_slots;
  int validate;
  unsigned int *status;
};

// Launchers (return cudaGetLastError() of the launch).
cudaError_t launch_prefill_simt(const PrefillParams &p, kda_dtype in_dtype, kda_dtype out_dtype,
                                cudaStream_t stream);
cudaError_t launch_prefill_tc(const PrefillParams &p, kda_dtype in_dtype, kda_dtype out_dtype,
                              cudaStream_t stream);
bool prefill_tc_supported(int dk, int dv, kda_dtype in_dtype);
int prefill_simt_slices(int dk, int dv, bool local_mode);
cudaError_t launch_schedule(const int32_t *cu_seqlens, int n_req, int32_t *order,
                            cudaStream_t stream);
cudaError_t launch_decode(const DecodeParams &p, kda_dtype in_dtype, kda_dtype out_dtype,
                          cudaStream_t stream);
cudaError_t launch_combine(const float *s_loc, const float *m, const float *s_init, int n_seg,
                           int H, int dk, int dv, float *s_in, float *s_final,
                           cudaStream_t stream);
unsigned int *device_status_word();  // address of the current device's status word

// Device address of a __device__ symbol of this library on the current device,
// cached per device and context under a lock (kda_api.cu).
class SymbolAddressCache {
 public:
  explicit SymbolAddressCache(const void *symbol);
  void *get();  // NULL if no device is usable

 private:
  const void *symbol_;
  std::mutex mu_;
  CUcontext ctx_[64] = {};
  void *addr_[64] = {};
};

// Backward of the prefill (kda_backward.cu).  The workspace holds, in order,
// the chunk table, the chunk-start snapshots of a forward pass, a zero state
// and the per-(chunk, head) intermediates; backward_offsets() gives the first
// five regions so the host can fill the tables and run the forward pass.
struct BackwardLaunch {
  const void *q, *k, *v;
  const float *g, *beta, *initial_state, *d_o, *d_final;
  const __nv_bfloat16 *g_logits;  // when set (g NULL), dg is the gradient of the logits
  float *dq, *dk, *dv, *dg, *dbeta, *d_initial;
  void *workspace;
  int n_req, n_chunks, n_snap, H, D;
  kda_dtype in_dtype;
};
cudaError_t launch_backward(const BackwardLaunch &b, cudaStream_t stream);
size_t backward_workspace_bytes(int n_req, int n_chunks, int n_snap, int H, int D);
void backward_offsets(int n_req, int n_chunks, int n_snap, int H, int D, size_t *chunks,
                      size_t *cu_chunks, size_t *cu_snap, size_t *snaps, size_t *zero);

// Fused gate activation: the lower-bounded decay log(alpha) = -5 sigmoid(x) of a
// gate logit x, which lies in [-5, 0] for every x (alpha >= exp(-5)), and its
// derivative d log(alpha) / dx = -5 sigmoid(x) (1 - sigmoid(x)).  The sigmoid is
// 1 / (1 + 2^(-x log2 e)) with the approximate ex2 and rcp instructions (relative
// error a few 1e-7); for x below about -88 the power is +inf and the gate is 0, the
// limit.
__device__ __forceinline__ float gate_sigmoid(float x) {
  float e, r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(-1.4426950408889634f * x));
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(1.f + e));
  return r;
}
__device__ __forceinline__ float gate_from_logit(float x) { return kGateLower * gate_sigmoid(x); }
__device__ __forceinline__ float gate_logit_slope(float x) {
  const float s = gate_sigmoid(x);
  return kGateLower * s * (1.f - s);
}

// Element loads/stores shared by the kernels.
__device__ __forceinline__ float load_elem(const float *p, size_t i) { return p[i]; }
__device__ __forceinline__ float load_elem(const __nv_bfloat16 *p, size_t i) {
  return __bfloat162float(p[i]);
}
__device__ __forceinline__ void store_elem(float *p, size_t i, float x) { p[i] = x; }
__device__ __forceinline__ void store_elem(__nv_bfloat16 *p, size_t i, float x) {
  p[i] = __float2bfloat16_rn(x);
}

}  // namespace kda

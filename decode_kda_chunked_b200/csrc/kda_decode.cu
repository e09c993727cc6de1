// KDA decode step (sm_100a): one new token per request against its
// fixed-size fp32 state ("Kimi K3 开源日来了", Infra section, second layer:
// KDA keeps one fixed-size recurrent state per request).
//
// Per (request, head), with S the dk x dv state of the request's slot:
//   S' = Diag(alpha) S;  u = S'^T k;  r = S'^T q  (one pass over S)
//   delta = beta (v - u);  o = r + (k . q) delta;  S <- S' + k delta^T
// which is S <- (I - beta k k^T) Diag(alpha) S + beta k v^T followed by
// o = S^T q, rearranged so the state is read once and written once.
//
// The step is bound by HBM: 2 * dk * dv * 4 bytes of state traffic against
// about 7 * dk * dv flops.  One CTA owns one state; each thread keeps its
// rows x 4 columns of the state in registers between the read and the
// write, and every global access is a coalesced 16-byte vector.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float4 ld_stream(const float4 *p) { return __ldcs(p); }
__device__ __forceinline__ void st_stream(float4 *p, float4 v) { __stcs(p, v); }

template <int D, typename TIn, typename TOut>
__global__ void __launch_bounds__(kThreads, 2) decode_kernel(const DecodeParams p) {
  constexpr int CG = D / 4;             // float4 column groups per row
  constexpr int RG = kThreads / CG;     // row groups
  constexpr int RPT = D / RG;           // rows per thread
  static_assert(RPT * RG == D, "row split");

  __shared__ float s_ak[D], s_aq[D], s_a[D], s_k[D];
  __shared__ float s_red_u[RG][D], s_red_r[RG][D];
  __shared__ float s_delta[D];
  __shared__ float s_kq;

  const int tid = threadIdx.x;
  const int nh = blockIdx.x;
  const int n = nh / p.H, h = nh % p.H;
  const int slot_raw = p.slot ? p.slot[n] : n;
  const bool slot_ok = slot_raw >= 0 && slot_raw < p.n_slots;
  const int slot = slot_ok ? slot_raw : 0;  // never touch memory outside the pool
  float *S = p.state + ((size_t)slot * p.H + h) * D * D;
  const size_t tok = (size_t)n * p.H + h;

  const int cg = tid % CG, rg = tid / CG;
  // The token's few values first, then the state: every load of the step is in
  // flight at once, so the token reads (fresh every step) hide under the state stream.
  float kk = 0.f, qq = 0.f, gg = 0.f, vv = 0.f, bb = 0.f;
  if (tid < D) {
    kk = load_elem(static_cast<const TIn *>(p.k), tok * D + tid);
    qq = load_elem(static_cast<const TIn *>(p.q), tok * D + tid);
    gg = p.g[tok * D + tid];
    vv = load_elem(static_cast<const TIn *>(p.v), tok * D + tid);
    bb = p.beta[tok];
  }
  float4 s[RPT];
#pragma unroll
  for (int rr = 0; rr < RPT; ++rr)
    s[rr] = ld_stream(reinterpret_cast<const float4 *>(S + (size_t)(rg * RPT + rr) * D) + cg);
  if (!slot_ok) {  // uniform per CTA: report and write nothing
    if (tid == 0) set_status(p.status, STATUS_BAD_SEQLENS);
    return;
  }

  if (tid < D) {
    if (p.validate && !(gg >= kGateLower && gg <= 0.f)) set_status(p.status, STATUS_GATE_RANGE);
    const float a = expf(gg);
    s_a[tid] = a;
    s_k[tid] = kk;
    s_ak[tid] = a * kk;
    s_aq[tid] = a * qq;
    // k . q, reduced by the first D/32 warps through shared memory below
    float kq = kk * qq;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);
    if ((tid & 31) == 0) s_red_u[0][tid >> 5] = kq;  // scratch, overwritten later
  }
  __syncthreads();
  if (tid == 0) {
    float kq = 0.f;
    for (int w = 0; w < D / 32; ++w) kq += s_red_u[0][w];
    s_kq = kq;
  }
  __syncthreads();

  // partial u = S'^T k and r = S'^T q over this thread's rows
  float4 pu = make_float4(0.f, 0.f, 0.f, 0.f), pr = pu;
#pragma unroll
  for (int rr = 0; rr < RPT; ++rr) {
    const int i = rg * RPT + rr;
    const float ak = s_ak[i], aq = s_aq[i];
    pu.x = fmaf(ak, s[rr].x, pu.x); pu.y = fmaf(ak, s[rr].y, pu.y);
    pu.z = fmaf(ak, s[rr].z, pu.z); pu.w = fmaf(ak, s[rr].w, pu.w);
    pr.x = fmaf(aq, s[rr].x, pr.x); pr.y = fmaf(aq, s[rr].y, pr.y);
    pr.z = fmaf(aq, s[rr].z, pr.z); pr.w = fmaf(aq, s[rr].w, pr.w);
  }
  *reinterpret_cast<float4 *>(&s_red_u[rg][4 * cg]) = pu;
  *reinterpret_cast<float4 *>(&s_red_r[rg][4 * cg]) = pr;
  __syncthreads();

  if (tid < D) {
    float u = 0.f, rr_ = 0.f;
#pragma unroll
    for (int g = 0; g < RG; ++g) {
      u += s_red_u[g][tid];
      rr_ += s_red_r[g][tid];
    }
    if (p.validate && !(bb >= 0.f && bb <= 1.f)) set_status(p.status, STATUS_GATE_RANGE);
    const float delta = bb * (vv - u);
    s_delta[tid] = delta;
    store_elem(static_cast<TOut *>(p.o), tok * D + tid, fmaf(s_kq, delta, rr_));
  }
  __syncthreads();

  const float4 d4 = *reinterpret_cast<const float4 *>(&s_delta[4 * cg]);
#pragma unroll
  for (int rr = 0; rr < RPT; ++rr) {
    const int i = rg * RPT + rr;
    const float a = s_a[i], kk = s_k[i];
    float4 o;
    o.x = fmaf(kk, d4.x, a * s[rr].x);
    o.y = fmaf(kk, d4.y, a * s[rr].y);
    o.z = fmaf(kk, d4.z, a * s[rr].z);
    o.w = fmaf(kk, d4.w, a * s[rr].w);
    st_stream(reinterpret_cast<float4 *>(S + (size_t)i * D) + cg, o);
  }
}

template <int D, typename TIn>
cudaError_t launch_d(const DecodeParams &p, kda_dtype out_dtype, cudaStream_t stream) {
  const long long blocks = (long long)p.n * p.H;
  if (blocks == 0) return cudaSuccess;
  if (out_dtype == KDA_BF16)
    decode_kernel<D, TIn, __nv_bfloat16><<<(unsigned)blocks, kThreads, 0, stream>>>(p);
  else
    decode_kernel<D, TIn, float><<<(unsigned)blocks, kThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const DecodeParams &p, kda_dtype in_dtype, kda_dtype out_dtype,
                          cudaStream_t stream) {
  if (p.dk == 128) {
    if (in_dtype == KDA_BF16) return launch_d<128, __nv_bfloat16>(p, out_dtype, stream);
    return launch_d<128, float>(p, out_dtype, stream);
  }
  if (in_dtype == KDA_BF16) return launch_d<64, __nv_bfloat16>(p, out_dtype, stream);
  return launch_d<64, float>(p, out_dtype, stream);
}

}  // namespace kda

// Segment combine and work scheduling (sm_100a).
//
// Combine: the exchange step of KDA context parallelism ("Kimi K3 开源日来了",
// Infra section, first layer: every segment's true start state is recovered
// exactly from each segment's zero-start state S_loc and transition M):
//     S_in[0] = S_init,  S_in[s+1] = M[s] S_in[s] + S_loc[s].
// The scan is serial over segments; columns of the state are independent, so
// one CTA owns (head, 16-column slice) and keeps its slice of the running
// state in shared memory while M[s] streams through shared memory.
//
// Schedule: orders requests longest first so the longest serial chains of
// the chunked prefill start earliest (the order never changes results).
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kThreads = 256;
constexpr int kCols = 16;

template <int DK>
__global__ void __launch_bounds__(kThreads) combine_kernel(const float *__restrict__ s_loc,
                                                           const float *__restrict__ m,
                                                           const float *__restrict__ s_init,
                                                           int n_seg, int H, int dv,
                                                           float *__restrict__ s_in,
                                                           float *__restrict__ s_final) {
  extern __shared__ float4 smem_f4[];
  float *sM = reinterpret_cast<float *>(smem_f4);  // [DK][DK]
  float *cur = sM + DK * DK;                        // [DK][kCols]
  const int slices = dv / kCols;
  const int h = blockIdx.x / slices, col0 = (blockIdx.x % slices) * kCols;
  const int tid = threadIdx.x;
  const int j = tid % kCols, i0 = tid / kCols;      // thread owns rows i0 + 16*ii
  constexpr int RN = DK / (kThreads / kCols);

  for (int idx = tid; idx < DK * kCols; idx += kThreads) {
    const int i = idx / kCols, jj = idx % kCols;
    cur[idx] = s_init ? s_init[((size_t)h * DK + i) * dv + col0 + jj] : 0.f;
  }
  for (int s = 0; s < n_seg; ++s) {
    const size_t base = (size_t)s * H + h;
    const float4 *Ms = reinterpret_cast<const float4 *>(m + base * DK * DK);
    __syncthreads();  // cur complete, previous M consumed
    for (int idx = tid; idx < DK * DK / 4; idx += kThreads)
      reinterpret_cast<float4 *>(sM)[idx] = Ms[idx];
    if (s_in)
      for (int idx = tid; idx < DK * kCols; idx += kThreads) {
        const int i = idx / kCols, jj = idx % kCols;
        s_in[(base * DK + i) * dv + col0 + jj] = cur[idx];
      }
    __syncthreads();
    float acc[RN];
#pragma unroll
    for (int ii = 0; ii < RN; ++ii) {
      const int i = i0 + (kThreads / kCols) * ii;
      acc[ii] = s_loc[(base * DK + i) * dv + col0 + j];
    }
    for (int l = 0; l < DK; ++l) {
      const float b = cur[l * kCols + j];
#pragma unroll
      for (int ii = 0; ii < RN; ++ii) {
        const int i = i0 + (kThreads / kCols) * ii;
        acc[ii] = fmaf(sM[i * DK + l], b, acc[ii]);
      }
    }
    __syncthreads();  // everyone has read cur
#pragma unroll
    for (int ii = 0; ii < RN; ++ii) {
      const int i = i0 + (kThreads / kCols) * ii;
      cur[i * kCols + j] = acc[ii];
    }
  }
  __syncthreads();
  if (s_final)
    for (int idx = tid; idx < DK * kCols; idx += kThreads) {
      const int i = idx / kCols, jj = idx % kCols;
      s_final[((size_t)h * DK + i) * dv + col0 + jj] = cur[idx];
    }
}

// rank of request r = number of requests that go before it (longer, or equal
// length and lower index); order[rank] = r.  O(n^2) work spread over n threads.
__global__ void schedule_kernel(const int32_t *__restrict__ cu, int n_req,
                                int32_t *__restrict__ order) {
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= n_req) return;
  const int lr = cu[r + 1] - cu[r];
  int rank = 0;
  for (int q = 0; q < n_req; ++q) {
    const int lq = cu[q + 1] - cu[q];
    rank += (lq > lr) || (lq == lr && q < r);
  }
  order[rank] = r;
}

}  // namespace

cudaError_t launch_combine(const float *s_loc, const float *m, const float *s_init, int n_seg,
                           int H, int dk, int dv, float *s_in, float *s_final,
                           cudaStream_t stream) {
  const unsigned blocks = (unsigned)(H * (dv / kCols));
  if (blocks == 0) return cudaSuccess;
  if (dk == 128) {
    const size_t bytes = sizeof(float) * (128 * 128 + 128 * kCols);
    cudaError_t e = cudaFuncSetAttribute(combine_kernel<128>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return e;
    combine_kernel<128><<<blocks, kThreads, bytes, stream>>>(s_loc, m, s_init, n_seg, H, dv,
                                                             s_in, s_final);
  } else {
    const size_t bytes = sizeof(float) * (64 * 64 + 64 * kCols);
    combine_kernel<64><<<blocks, kThreads, bytes, stream>>>(s_loc, m, s_init, n_seg, H, dv, s_in,
                                                            s_final);
  }
  return cudaGetLastError();
}

cudaError_t launch_schedule(const int32_t *cu_seqlens, int n_req, int32_t *order,
                            cudaStream_t stream) {
  if (n_req <= 0) return cudaSuccess;
  const int threads = 256;
  schedule_kernel<<<(n_req + threads - 1) / threads, threads, 0, stream>>>(cu_seqlens, n_req,
                                                                         order);
  return cudaGetLastError();
}

}  // namespace kda

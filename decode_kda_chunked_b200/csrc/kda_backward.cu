// KDA backward (training) on sm_100a: gradients of the chunked prefill.
//
// FlashKDA also speeds up training ("Kimi K3 开源日来了", FlashKDA section), so
// the path carries the derivative of the prefill map: given cotangents dO of o
// and dS_L of the final state, the gradients of q, k, v, g (= log alpha),
// beta and the initial state.
//
// Reverse mode through the forward's chunk algebra (one chain; chunk start
// state S, chunk-end cotangent dSn, G the chunk-local cumsum of g,
// gamma = exp(G), Gam = gamma at the chunk's last row, Khat = (Gam/gamma) K,
// [U~ | W] = T Diag(beta) [V | gamma K], U = U~ - W S, T = (I + Diag(beta) A)^-1):
//
//   serial over chunks, last to first:
//     dU = P^T dO + Khat dSn
//     dS = Diag(Gam) dSn + (gamma Q)^T dO - W^T dU
//   per chunk, all chunks in parallel:
//     d(gamma Q) = dO S^T      dP = tril(dO U^T)      dKhat = U dSn^T      dW = -dU S^T
//     dV = Diag(beta) T^T dU   d(gamma K) = Diag(beta) T^T dW
//     dT = dU (Diag(beta) V)^T + dW (Diag(beta) gamma K)^T, which T^-1 maps to
//     dZ = -T^T dT T^T = -[(T^T dU) U~^T + (T^T dW) W^T]   dA = tril_strict(Diag(beta) dZ)
//     dbeta_t = (T^T dU)_t . v_t + (T^T dW)_t . (gamma k)_t + sum_s dZ_ts A_ts
//     A and P are gated Gram products; their cotangents reach K, Q and the
//     cumulative gate through sums  sum_s M_ts x_s exp(G_t - G_s)  (t >= s),
//     each taken with the 16-row block factorisation
//     exp(G_t - G_s) = exp(G_t - G_r) exp(G_r - G_s), r a block boundary, so
//     every factor is a finite fp32 number (log alpha >= -5, the lower-bounded
//     decay of KDA, CSDN post on the Kimi K3 technical report, section 一.1).
//     dg = reverse cumulative sum of dG over the chunk.
//
// Launches: the forward kernel with a snapshot every 64 tokens (the chunk
// start states), then
//   bwd_prep   (CTA per chunk and head): A, T, W, U~, Khat, Gam, X = P^T dO, Y = (gamma Q)^T dO
//   bwd_state  the serial pass; dU overwrites X, dSn overwrites Y.  bwd_state_tc (CTA
//              per request and head; bf16 inputs at d = 128) on the tensor cores with
//              dS^T in TMEM, else bwd_state (CTA per request, head and 32 state columns)
//   bwd_sprod  (CTA per chunk and head; bf16 inputs at d = 128): on the tensor cores,
//              U, d(gamma Q), dKhat, dW and dGam (the products with the state), then
//              dP, T^T dU, T^T dW and dZ (the products of chunk-sized tiles)
//   bwd_grad   (CTA per chunk and head): every token gradient of the chunk
// For bf16 inputs at d = 128 every dense product runs as tcgen05 tf32 MMAs (transposed
// to M = 128 TMEM lanes, as in the forward), the gated Gram cotangents of bwd_grad
// included, and the CUDA cores keep the per-element folds; fp32 inputs keep fp32
// products on the CUDA cores throughout.  The CUDA-core passes give thread (ty, tx) of a 16 x TX grid rows
// ty + 16 i and columns tx + TX j of every tile it produces, so per-element folds stay
// in registers.
#include "kda_internal.cuh"
#include "kda_sm100.cuh"

#include <type_traits>

namespace kda {

namespace {

using namespace sm100;

constexpr int NTH = 256;
constexpr int C = kChunk;  // 64
constexpr float LOG2E = 1.4426950408889634f;

struct BwdParams {
  const void *q, *k, *v;
  const float *g, *beta;
  const __nv_bfloat16 *g_logits;  // when set (g NULL): log alpha = -5 sigmoid(logit), and dg
                                  // is the gradient of the logits
  const float *initial_state;  // NULL = zeros
  const float *d_o;            // NULL = zeros
  const float *d_final;        // NULL = zeros
  float *dq, *dk, *dv, *dg, *dbeta;
  float *d_initial;            // NULL = not returned
  const int4 *chunks;          // per chunk: request, chunk index in the request, first token, rows
  const int32_t *cu_chunks;    // [n_req + 1]
  const int32_t *cu_snap;      // [n_req + 1]: chunk-start snapshots of the forward pass
  const float *snaps;          // [n_snap, H, D, D]
  const float *zero_state;     // D x D zeros
  float *wA, *wT, *wW, *wU, *wKh, *wX, *wY, *wGam;
  float *wU2;                  // per (chunk, head): U = U~ - W S from the gradient pass (fp32
                               // inputs), or dZ from bwd_sprod (bf16 inputs at d = 128)
  int n_req, n_chunks, H;
  unsigned int *status;        // device status word (a bounded wait that gave up)
};

// acc[i][j] += sum_k A(m_i, k) B(k, n_j) for k < K (a multiple of 16), where
// the calling thread's rows are m_i = ty + 16 i and columns n_j = tx + 16 j;
// A(m, k) = A[m am + k ak], B(k, n) = B[k bk + n bn], in any memory space.
// Slices of 16 along k are staged through shared memory `stage`
// (16 (16 MI + 1) + 16 (16 NJ + 1) floats) so the inner loop reads
// conflict-free shared memory; the next slice is loaded into registers while
// the current one is multiplied.  Every thread of the CTA must call it; it
// synchronises the CTA before its first load, so operands written by the CTA
// just before the call are complete.
template <int MI, int NJ>
__device__ void mm_acc(float (&acc)[MI][NJ], const float *A, int am, int ak, const float *B,
                       int bk, int bn, int K, float *stage) {
  static_assert(MI % 4 == 0 && NJ % 4 == 0, "rows and columns load as float4 runs");
  constexpr int M = 16 * MI, N = 16 * NJ;
  // Staged slices are stored permuted so a thread's MI rows (ty + 16 i) and NJ columns
  // (tx + 16 j) sit side by side: row m at MI (m % 16) + m / 16; column n at
  // NJ (n % 16) + n / 16, plus 4 floats per group of four threads when NJ = 8, which
  // keeps every quarter-warp's 16-byte loads on distinct banks.
  constexpr int PADB = NJ >= 8 ? 4 : 0;
  constexpr int LA = M + 4, LB = N + 4 * PADB + 4;
  float *As = stage, *Bs = stage + 16 * LA;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  // each thread moves MI elements of the A slice and NJ of the B slice; the
  // walk order puts consecutive threads on the operand's contiguous axis
  const bool a_k_inner = ak == 1, b_n_inner = bn == 1;
  auto a_at = [&](int e, int &kk, int &m) {
    if (a_k_inner) { kk = e & 15; m = e >> 4; } else { m = e % M; kk = e / M; }
  };
  auto b_at = [&](int e, int &kk, int &n) {
    if (b_n_inner) { n = e % N; kk = e / N; } else { kk = e & 15; n = e >> 4; }
  };
  auto a_pos = [&](int m) { return MI * (m & 15) + (m >> 4); };
  auto b_pos = [&](int n) { return NJ * (n & 15) + (n >> 4) + PADB * ((n & 15) >> 2); };
  float ra[MI], rb[NJ];
  auto fetch = [&](int k0) {
#pragma unroll
    for (int q = 0; q < MI; ++q) {
      int kk, m;
      a_at(tid + q * NTH, kk, m);
      ra[q] = A[(size_t)m * am + (size_t)(k0 + kk) * ak];
    }
#pragma unroll
    for (int q = 0; q < NJ; ++q) {
      int kk, n;
      b_at(tid + q * NTH, kk, n);
      rb[q] = B[(size_t)(k0 + kk) * bk + (size_t)n * bn];
    }
  };
  const int a_base = MI * ty, b_base = NJ * tx + PADB * (tx >> 2);
  __syncthreads();  // operands the CTA has just written are complete before the first fetch
  fetch(0);
  for (int k0 = 0; k0 < K; k0 += 16) {
    __syncthreads();  // the previous slice has been consumed
#pragma unroll
    for (int q = 0; q < MI; ++q) {
      int kk, m;
      a_at(tid + q * NTH, kk, m);
      As[kk * LA + a_pos(m)] = ra[q];
    }
#pragma unroll
    for (int q = 0; q < NJ; ++q) {
      int kk, n;
      b_at(tid + q * NTH, kk, n);
      Bs[kk * LB + b_pos(n)] = rb[q];
    }
    __syncthreads();
    if (k0 + 16 < K) fetch(k0 + 16);  // next slice in flight during this one's FMAs
#pragma unroll 4
    for (int kk = 0; kk < 16; ++kk) {
      float a[MI], b[NJ];
#pragma unroll
      for (int q = 0; q < MI / 4; ++q)
        *reinterpret_cast<float4 *>(&a[4 * q]) =
            *reinterpret_cast<const float4 *>(As + kk * LA + a_base + 4 * q);
#pragma unroll
      for (int q = 0; q < NJ / 4; ++q)
        *reinterpret_cast<float4 *>(&b[4 * q]) =
            *reinterpret_cast<const float4 *>(Bs + kk * LB + b_base + 4 * q);
#pragma unroll
      for (int i = 0; i < MI; ++i)
#pragma unroll
        for (int j = 0; j < NJ; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
  }
  __syncthreads();
}

template <int MI, int NJ>
__device__ __forceinline__ void zero(float (&acc)[MI][NJ]) {
#pragma unroll
  for (int i = 0; i < MI; ++i)
#pragma unroll
    for (int j = 0; j < NJ; ++j) acc[i][j] = 0.f;
}

// shared floats mm_acc stages for an M x N output (the padded A and B slices)
constexpr int stage_floats(int M, int N) { return 16 * (M + 4) + 16 * (N + 4 * (N >= 128 ? 4 : 0) + 4); }

// Rows tok0 .. tok0 + n - 1 of a token-major [T, H, D] tensor into a [64][ld]
// fp32 tile (rows >= n are zero: the exact no-op padding of the chunk form).
// 16-byte loads, all of a thread's loads issued before any of its stores.
__device__ __forceinline__ void unpack16(const uint4 &u, const float *, float (&x)[4]) {
  x[0] = __uint_as_float(u.x); x[1] = __uint_as_float(u.y);
  x[2] = __uint_as_float(u.z); x[3] = __uint_as_float(u.w);
}
__device__ __forceinline__ void unpack16(const uint4 &u, const __nv_bfloat16 *, float (&x)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    x[2 * q] = __uint_as_float(w[q] << 16);
    x[2 * q + 1] = __uint_as_float(w[q] & 0xFFFF0000u);
  }
}
template <int D, typename TIn, int NT = NTH>
__device__ void stage_rows(float *dst, int ld, const TIn *src, int tok0, int n, int H, int h) {
  constexpr int VEC = 16 / (int)sizeof(TIn);  // elements per 16-byte load
  constexpr int PER_ROW = D / VEC, ITER = C * PER_ROW / NT;
  static_assert(ITER * NT == C * PER_ROW, "tile must split evenly over the CTA");
  uint4 buf[ITER];
#pragma unroll
  for (int it = 0; it < ITER; ++it) {
    const int e = threadIdx.x + it * NT, t = e / PER_ROW, cv = e % PER_ROW;
    buf[it] = (src && t < n)
                  ? *reinterpret_cast<const uint4 *>(src + ((size_t)(tok0 + t) * H + h) * D + cv * VEC)
                  : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int it = 0; it < ITER; ++it) {
    const int e = threadIdx.x + it * NT, t = e / PER_ROW, cv = e % PER_ROW;
    float x[VEC];
    unpack16(buf[it], src, x);
    if ((ld & 3) == 0) {  // 16-byte aligned rows: vector stores
#pragma unroll
      for (int q = 0; q < VEC / 4; ++q)
        *reinterpret_cast<float4 *>(dst + t * ld + cv * VEC + 4 * q) =
            make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
    } else {
#pragma unroll
      for (int q = 0; q < VEC; ++q) dst[t * ld + cv * VEC + q] = x[q];
    }
  }
}

// g rows into sG, then the in-place chunk-local cumsum scaled by log2(e)
// (thread = channel); beta into sB.  Padded rows have g = 0 and beta = 0.
template <int D, int NT = NTH>
__device__ void stage_gate(float *sG, float *sB, const BwdParams &p, int tok0, int n, int h,
                           int ld = D) {
  if (p.g_logits)
    stage_rows<D, __nv_bfloat16, NT>(sG, ld, p.g_logits, tok0, n, p.H, h);
  else
    stage_rows<D, float, NT>(sG, ld, p.g, tok0, n, p.H, h);
  if (threadIdx.x < C)
    sB[threadIdx.x] = threadIdx.x < n ? p.beta[(size_t)(tok0 + threadIdx.x) * p.H + h] : 0.f;
  __syncthreads();
  if (threadIdx.x < D) {
    const int c = threadIdx.x;
    float run = 0.f;
    if (p.g_logits) {
      for (int t = 0; t < C; ++t) {
        run += t < n ? gate_from_logit(sG[t * ld + c]) : 0.f;
        sG[t * ld + c] = run * LOG2E;
      }
    } else {
      for (int t = 0; t < C; ++t) {
        run += sG[t * ld + c];
        sG[t * ld + c] = run * LOG2E;
      }
    }
  }
  __syncthreads();
}

// Gate tables store a row's column c at a permuted position so the thread that owns
// columns tx + TX j (j < NJ) reads them as NJ / 4 float4 chunks (2 tx, 2 tx + 1 for
// NJ = 8 at TX = 16, with chunk bit 0 flipped by tx bit 2 so every quarter-warp covers
// all 32 banks; chunk tx for NJ = 4).
template <int TX, int NJ>
__device__ __forceinline__ int gate_pos(int c) {
  const int tx = c % TX, j = c / TX;
  if (NJ == 8) return 4 * ((2 * tx + (j >> 2)) ^ ((tx >> 2) & 1)) + (j & 3);
  return 4 * tx + j;
}
template <int TX, int NJ>
__device__ __forceinline__ int gate_chunk(int tx, int q) {
  return NJ == 8 ? ((2 * tx + q) ^ ((tx >> 2) & 1)) : tx;
}

// Sum over the TX lanes that share a row (TX = 16: one half-warp; 32: the warp).
template <int TX>
__device__ __forceinline__ float row_sum(float x) {
#pragma unroll
  for (int off = TX / 2; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}

// ---------------------------------------------------------------------------
// bwd_prep: the state-independent chunk quantities
// ---------------------------------------------------------------------------
template <int D>
struct PrepLayout {
  // Row strides: LDP for the scratch tiles; the k, q and g tiles take D + 1 and the A and
  // P tiles C + 1 (kernels that read them with one lane per row then hit distinct banks)
  static constexpr int LDP = D + 1, LK = D + 1, LA = C + 1;
  static constexpr int oK = 0, oQ = oK + C * LK, oG = oQ + C * LK;
  static constexpr int oA = (oG + C * LK + 255) / 256 * 256;  // keeps oBuf 1024-byte aligned
  static constexpr int oP = oA + C * LA, oT = oP + C * LA, oBuf = oT + C * C + 128;
  static constexpr int oKL = oBuf + C * LDP, oQL = oKL + 16 * LDP, oStage = oQL + 16 * LDP;
  static constexpr int oB = oStage + stage_floats(D, D);
  static constexpr int oMisc = oB + C;  // two mbarriers (8 bytes each) and the TMEM base address
  static constexpr int total = oMisc + 6;
  // + alignment slack: the tensor-core operand tiles need a 1024-byte aligned base
  static constexpr size_t bytes = sizeof(float) * total + 1024;
};

// The products of the prep pass run on the tensor cores (tf32, like the forward's)
// for bf16 inputs at d = 128; fp32 inputs keep fp32 products (their 1e-5 tolerance
// rules out tf32 operands).
template <int D, typename TIn>
constexpr bool kPrepTensorCores = D == 128 && std::is_same<TIn, __nv_bfloat16>::value;

// Threads of the gradient pass: 512 (16 x 32, four columns of d = 128 per thread) when
// its dense products come from the tensor cores, else 256 (16 x 16, for the fp32 tile
// products it then runs itself).
template <int D, typename TIn>
__host__ __device__ constexpr int grad_threads() { return kPrepTensorCores<D, TIn> ? 512 : 256; }

// Threads of the prep pass: 512 when its products run on the tensor cores (16 warps
// share the operand staging, the read-out and the triangular solve), else 256 (its
// fp32 tile products assume a 16 x 16 thread grid).
template <int D, typename TIn>
__host__ __device__ constexpr int prep_threads() { return kPrepTensorCores<D, TIn> ? 512 : 256; }

// fp32 -> tf32, round to nearest even (the tensor cores read the 19 leading bits)
__device__ __forceinline__ float tf32_round(float x) {
  uint32_t r;
  asm("cvt.rn.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}
__device__ __forceinline__ float4 tf32_round4(float4 x) {
  return make_float4(tf32_round(x.x), tf32_round(x.y), tf32_round(x.z), tf32_round(x.w));
}

template <int D, typename TIn>
__global__ void __launch_bounds__(prep_threads<D, TIn>(), 1) bwd_prep_kernel(const BwdParams p) {
  using L = PrepLayout<D>;
  constexpr int NJ = D / 16, LDP = L::LDP, LK = L::LK, LA = L::LA, PN = prep_threads<D, TIn>();
  extern __shared__ float4 smem_f4[];
  float *sm = reinterpret_cast<float *>(align1024_shared(smem_f4));
  float *sK = sm + L::oK, *sQ = sm + L::oQ, *sG = sm + L::oG, *sA = sm + L::oA;
  float *sP = sm + L::oP, *sT = sm + L::oT, *sBuf = sm + L::oBuf, *sKL = sm + L::oKL;
  float *sQL = sm + L::oQL, *sStage = sm + L::oStage, *sB = sm + L::oB;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const int H = p.H;
  const int jc = blockIdx.x / H, h = blockIdx.x % H;
  const int4 cd = p.chunks[jc];
  const int tok0 = cd.z, n = cd.w;
  const size_t ch = (size_t)jc * H + h;
  uint64_t *bar = reinterpret_cast<uint64_t *>(sm + L::oMisc);  // [0]: products, [1]: A|P
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(sm + L::oMisc + 4);
  if constexpr (kPrepTensorCores<D, TIn>) {
    if ((tid >> 5) == 0) {
      tmem_alloc(s_tmem, 512);
      tmem_relinquish();
    }
    if (tid == 0) {
      mbar_init(bar, 1);
      mbar_init(bar + 1, 1);
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
  }
  bool ap_done = true;

  stage_rows<D, TIn, PN>(sK, LK, static_cast<const TIn *>(p.k), tok0, n, H, h);
  stage_rows<D, TIn, PN>(sQ, LK, static_cast<const TIn *>(p.q), tok0, n, H, h);
  stage_gate<D, PN>(sG, sB, p, tok0, n, h, LK);

  if constexpr (kPrepTensorCores<D, TIn>) {
    // A and P on the tensor cores, as in the forward: two 32-row blocks b with reference
    // rows m_b = 32 b + 15; L*_i = x_i exp(G_i - G_mb) (<= e^75) in TMEM, lanes 0..63 the
    // k rows and 64..127 the q rows; R'_b row j = k_j exp(G_mb - G_j) (<= e^80, rows
    // j < 32 (b + 1)) as B operands in the scratch region; each block's product runs as two
    // 8-step chains over the key-channel halves, summed on read-out.  Masked entries
    // (s > t) may overflow and are dropped by selection.
    constexpr uint32_t TL = 0, TAP = 128;
    auto apc = [](int b, int hh) { return TAP + (b == 0 ? 32u * hh : 64u + 64u * hh); };
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = *s_tmem;
    const int w = tid >> 5, ln = tid & 31;
    const uint32_t lane = (uint32_t)(32 * (w & 3)) << 16;
    const int lr = 32 * (w & 3) + ln, i = lr & 63, m = 32 * (i >> 5) + 15;
    unsigned char *rp = reinterpret_cast<unsigned char *>(sBuf);  // 1024-byte aligned
    {  // warp w: lane quarter w % 4, channels 32 (w / 4) .. + 31
      const float *x = lr < C ? sK : sQ;
      const int c0 = 32 * (w >> 2);
      float v[32];
#pragma unroll
      for (int jj = 0; jj < 32; ++jj) {
        const int c = c0 + jj;
        v[jj] = tf32_round(x[i * LK + c] * exp2f(sG[i * LK + c] - sG[m * LK + c]));
      }
      tmem_st32(tm + lane + TL + c0, v);
    }
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      const int rows = 32 * (b + 1), mb = 32 * b + 15;
      // consecutive threads take consecutive rows j (distinct banks on both sides)
      for (int e = tid; e < rows * (D / 4); e += PN) {
        const int j = e % rows, c = (e / rows) * 4;
        float4 r;
        r.x = tf32_round(sK[j * LK + c] * exp2f(sG[mb * LK + c] - sG[j * LK + c]));
        r.y = tf32_round(sK[j * LK + c + 1] * exp2f(sG[mb * LK + c + 1] - sG[j * LK + c + 1]));
        r.z = tf32_round(sK[j * LK + c + 2] * exp2f(sG[mb * LK + c + 2] - sG[j * LK + c + 2]));
        r.w = tf32_round(sK[j * LK + c + 3] * exp2f(sG[mb * LK + c + 3] - sG[j * LK + c + 3]));
        *reinterpret_cast<float4 *>(rp + 16384 * b + sw128_chunk(rows, j, c)) = r;
      }
    }
    tmem_wait_st();
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
      const uint32_t rb = smem_u32(rp);
#pragma unroll
      for (int st = 0; st < D / 16; ++st)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
#pragma unroll
          for (int b = 0; b < 2; ++b) {
            const int ks = (D / 16) * hh + st;
            mma_tf32_ts(tm + apc(b, hh), tm + TL + 8 * ks,
                        sw128_desc(rb + 16384 * b, 32 * (b + 1), ks), idesc_tf32(32 * (b + 1)),
                        st > 0);
          }
      mma_commit(bar + 1);
    }
    ap_done = mbar_wait(bar + 1, 0);
    if (!ap_done && tid == 0) set_status(p.status, STATUS_TIMEOUT);
    tc_fence_after();
    {  // row i (lane lr), columns 16 (w / 4) .. + 15: A for k rows, P for q rows
      const int b = i >> 5, cb = 16 * (w >> 2);
      float a0[16], a1[16];
      tmem_ld16(tm + lane + apc(b, 0) + cb, a0);
      tmem_ld16(tm + lane + apc(b, 1) + cb, a1);
      tmem_wait_ld();
      if (lr < C) {
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) sA[i * LA + cb + jj] = (cb + jj < i) ? a0[jj] + a1[jj] : 0.f;
      } else {
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) sP[i * LA + cb + jj] = (cb + jj <= i) ? a0[jj] + a1[jj] : 0.f;
      }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  } else {
    // A (strict lower) and P (inclusive lower), row block b at a time:
    // A_ts = sum_c [k_tc exp(G_tc - G_rc)] [k_sc exp(G_rc - G_sc)], r = 16 b.
    // Unrolled over b, so the thread's valid column groups (jj <= b) are fixed.
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int r0 = 16 * b, rows = r0 + 16;
      __syncthreads();
      for (int e = tid; e < rows * D; e += PN) {
        const int s = e / D, c = e % D;
        sBuf[s * LDP + c] = sK[s * LK + c] * exp2f(sG[r0 * LK + c] - sG[s * LK + c]);
      }
      for (int e = tid; e < 16 * D; e += PN) {
        const int t = e / D, c = e % D;
        const float f = exp2f(sG[(r0 + t) * LK + c] - sG[r0 * LK + c]);
        sKL[t * LDP + c] = sK[(r0 + t) * LK + c] * f;
        sQL[t * LDP + c] = sQ[(r0 + t) * LK + c] * f;
      }
      __syncthreads();
      float a[4] = {0.f, 0.f, 0.f, 0.f}, pp[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
      for (int c = 0; c < D; ++c) {
        const float kl = sKL[ty * LDP + c], ql = sQL[ty * LDP + c];
#pragma unroll
        for (int jj = 0; jj <= b; ++jj) {
          const float tv = sBuf[(tx + 16 * jj) * LDP + c];
          a[jj] = fmaf(kl, tv, a[jj]);
          pp[jj] = fmaf(ql, tv, pp[jj]);
        }
      }
      const int t = r0 + ty;
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const int s = tx + 16 * jj;
        sA[t * LA + s] = s < t ? a[jj] : 0.f;
        sP[t * LA + s] = s <= t ? pp[jj] : 0.f;
      }
    }
    __syncthreads();
  }
  // T = (I + Diag(beta) A)^-1, blocked.  (1) The four 16x16 diagonal blocks by forward
  // substitution: column task j = tid / SP (block j / 16), its SP = PN / 64 threads (4
  // or 8) split each row's sum and combine it with shuffles inside their aligned group.
  // (2) The blocks below the diagonal, one block diagonal d at a time:
  //     T_ab = -T_aa sum_{c=b}^{a-1} N_ac T_cb,  N = Diag(beta) A,  b = a - d,
  // on a 16 x 16 grid per 256 threads (with 512, the two halves take alternate blocks a).
  {
    constexpr int SP = PN / 64;
    const int task = tid / SP, part = tid % SP;
    const int o = 16 * (task >> 4), j = o + (task & 15);
    for (int i = o; i < o + 16; ++i) {
      float acc = 0.f;
      for (int s = j + part; s < i; s += SP) acc = fmaf(sA[i * LA + s], sT[s * C + j], acc);
#pragma unroll
      for (int off = 1; off < SP; off <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      if (part == 0) sT[i * C + j] = i < j ? 0.f : (i == j ? 1.f : -sB[i] * acc);
      __syncwarp();
    }
    for (int e = tid; e < C * C; e += PN)  // blocks above the diagonal
      if ((e / C) >> 4 < (e % C) >> 4) sT[e] = 0.f;
    float *Ys = sBuf;  // [3][16][17] scratch: N_a. T_.b of one block diagonal
    const int half = tid / NTH, sy = (tid % NTH) >> 4, sx = tid & 15;
    for (int d = 1; d < 4; ++d) {
      __syncthreads();
      for (int a = d + half; a < 4; a += PN / NTH) {
        const int bb = a - d, i = 16 * a + sy, jc = 16 * bb + sx;
        float y = 0.f;
        for (int s2 = 16 * bb; s2 < 16 * a; ++s2) y = fmaf(sA[i * LA + s2], sT[s2 * C + jc], y);
        Ys[(bb * 16 + sy) * 17 + sx] = sB[i] * y;
      }
      __syncthreads();
      for (int a = d + half; a < 4; a += PN / NTH) {
        const int bb = a - d, i = 16 * a + sy, jc = 16 * bb + sx;
        float t = 0.f;
        for (int r = 16 * a; r <= i; ++r) t = fmaf(sT[i * C + r], Ys[(bb * 16 + r - 16 * a) * 17 + sx], t);
        sT[i * C + jc] = -t;
      }
    }
  }
  __syncthreads();

  if constexpr (kPrepTensorCores<D, TIn>) {
    // Transposed, so every product has M = 128 TMEM lanes (one per channel):
    //   W^T = (beta gamma K)^T T^T,  U~^T = (beta V)^T T^T,  X^T = dO^T P,  Y^T = dO^T (gamma Q)
    // A operands in TMEM (lane = channel, column = token), B operands K-major with the
    // 128-byte swizzle in shared memory: T and P^T in the scratch tile, (gamma Q)^T in
    // the (now unused) row-factor / staging region.
    constexpr uint32_t TA1 = 0, TA2 = 64, TA3 = 128, TD1 = 192, TD2 = 256, TD3 = 320, TD4 = 384;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = *s_tmem;
    // warp w: lane quarter w % 4 (channel c), tokens 16 (w / 4) .. + 15
    const int w = tid >> 5, ln = tid & 31, c = 32 * (w & 3) + ln, j0 = 16 * (w >> 2);
    const uint32_t lane = (uint32_t)(32 * (w & 3)) << 16;
    stage_rows<D, TIn, PN>(sBuf, LDP, static_cast<const TIn *>(p.v), tok0, n, H, h);
    __syncthreads();
    {
      float v1[16], v2[16];
#pragma unroll
      for (int jj = 0; jj < 16; ++jj) {
        const int j = j0 + jj;
        v1[jj] = tf32_round(sB[j] * exp2f(sG[j * LK + c]) * sK[j * LK + c]);
        v2[jj] = tf32_round(sB[j] * sBuf[j * LDP + c]);
      }
      tmem_st16(tm + lane + TA1 + j0, v1);
      tmem_st16(tm + lane + TA2 + j0, v2);
    }
    __syncthreads();  // V read out of the scratch tile
    stage_rows<D, float, PN>(sBuf, LDP, p.d_o, tok0, n, H, h);
    __syncthreads();
    {
      float v3[16];
#pragma unroll
      for (int jj = 0; jj < 16; ++jj) v3[jj] = tf32_round(sBuf[(j0 + jj) * LDP + c]);
      tmem_st16(tm + lane + TA3 + j0, v3);
    }
    tmem_wait_st();
    __syncthreads();  // dO read out of the scratch tile: it takes the B tiles now
    unsigned char *bT = reinterpret_cast<unsigned char *>(sBuf);
    unsigned char *bP = bT + 64 * 64 * 4;
    unsigned char *bQ = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(sKL) + 1023) & ~uintptr_t(1023));
    // each thread writes one 16-byte chunk (four K values of one operand row); consecutive
    // threads take consecutive rows, so both the source reads and the swizzled stores
    // fall on distinct banks
    for (int e = tid; e < C * C / 4; e += PN) {
      // T (row a, K = b) straight from its rows: a warp's quarter reads and writes one
      // row's 128 bytes
      const int a = e >> 4, b0 = (e & 15) * 4;
      *reinterpret_cast<float4 *>(bT + sw128_chunk(C, a, b0)) =
          tf32_round4(*reinterpret_cast<const float4 *>(sT + a * C + b0));
      // P^T (row b = r, K = a)
      const int r = e & 63, k0 = (e >> 6) * 4;
      *reinterpret_cast<float4 *>(bP + sw128_chunk(C, r, k0)) = tf32_round4(
          make_float4(sP[k0 * LA + r], sP[(k0 + 1) * LA + r], sP[(k0 + 2) * LA + r],
                      sP[(k0 + 3) * LA + r]));
    }
    for (int e = tid; e < D * C / 4; e += PN) {  // (gamma Q)^T: row nn = channel, K = token
      const int nn = e % D, j0 = (e / D) * 4;
      float x[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) x[u] = exp2f(sG[(j0 + u) * LK + nn]) * sQ[(j0 + u) * LK + nn];
      *reinterpret_cast<float4 *>(bQ + sw128_chunk(D, nn, j0)) =
          tf32_round4(make_float4(x[0], x[1], x[2], x[3]));
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
      const uint32_t id64 = idesc_tf32(64), id128 = idesc_tf32(128);
      const uint32_t tb = smem_u32(bT), pb = smem_u32(bP), qb = smem_u32(bQ);
#pragma unroll
      for (int s = 0; s < C / 8; ++s) {
        mma_tf32_ts(tm + TD1, tm + TA1 + 8 * s, sw128_desc(tb, C, s), id64, s > 0);
        mma_tf32_ts(tm + TD2, tm + TA2 + 8 * s, sw128_desc(tb, C, s), id64, s > 0);
        mma_tf32_ts(tm + TD3, tm + TA3 + 8 * s, sw128_desc(pb, C, s), id64, s > 0);
        mma_tf32_ts(tm + TD4, tm + TA3 + 8 * s, sw128_desc(qb, D, s), id128, s > 0);
      }
      mma_commit(bar);
    }
    const bool done = mbar_wait(bar, 0);
    if (!done && tid == 0) set_status(p.status, STATUS_TIMEOUT);
    tc_fence_after();
    if (done) {
      float v[32];
      tmem_ld16(tm + lane + TD1 + j0, v);  // W[token][channel]
      tmem_wait_ld();
#pragma unroll
      for (int jj = 0; jj < 16; ++jj) p.wW[ch * C * D + (size_t)(j0 + jj) * D + c] = v[jj];
      tmem_ld16(tm + lane + TD2 + j0, v);  // U~
      tmem_wait_ld();
#pragma unroll
      for (int jj = 0; jj < 16; ++jj) p.wU[ch * C * D + (size_t)(j0 + jj) * D + c] = v[jj];
      tmem_ld16(tm + lane + TD3 + j0, v);  // X
      tmem_wait_ld();
#pragma unroll
      for (int jj = 0; jj < 16; ++jj) p.wX[ch * C * D + (size_t)(j0 + jj) * D + c] = v[jj];
      const int c0 = 32 * (w >> 2);  // Y[dk][dv] from Y^T (lane = dv), rows c0 .. + 31
      tmem_ld32(tm + lane + TD4 + c0, v);
      tmem_wait_ld();
#pragma unroll
      for (int jj = 0; jj < 32; ++jj) p.wY[ch * D * D + (size_t)(c0 + jj) * D + c] = v[jj];
    }
    tc_fence_before();
    __syncthreads();
    if (!done && tid == 0) mbar_wait(bar, 0, 100000000ull);  // give the products a last chance
    if (!ap_done && tid == 0) mbar_wait(bar + 1, 0, 100000000ull);  // and the A|P products
    __syncthreads();
    if (w == 0) {
      tc_fence_after();
      tmem_dealloc(tm, 512);
    }
  } else {
  float acc[4][NJ];
    // W = T Diag(beta) (gamma K)
    for (int e = tid; e < C * D; e += PN) {
      const int t = e / D, c = e % D;
      sBuf[t * LDP + c] = sB[t] * exp2f(sG[t * LK + c]) * sK[t * LK + c];
    }
    zero(acc);
    mm_acc<4, NJ>(acc, sT, C, 1, sBuf, LDP, 1, C, sStage);
  #pragma unroll
    for (int i = 0; i < 4; ++i)
  #pragma unroll
      for (int j = 0; j < NJ; ++j) p.wW[ch * C * D + (ty + 16 * i) * D + tx + 16 * j] = acc[i][j];
    // U~ = T Diag(beta) V
    stage_rows<D, TIn>(sBuf, LDP, static_cast<const TIn *>(p.v), tok0, n, H, h);
    __syncthreads();
    for (int e = tid; e < C * D; e += PN) sBuf[(e / D) * LDP + e % D] *= sB[e / D];
    zero(acc);
    mm_acc<4, NJ>(acc, sT, C, 1, sBuf, LDP, 1, C, sStage);
  #pragma unroll
    for (int i = 0; i < 4; ++i)
  #pragma unroll
      for (int j = 0; j < NJ; ++j) p.wU[ch * C * D + (ty + 16 * i) * D + tx + 16 * j] = acc[i][j];
    // X = P^T dO
    stage_rows<D, float>(sBuf, LDP, p.d_o, tok0, n, H, h);
    zero(acc);
    mm_acc<4, NJ>(acc, sP, 1, LA, sBuf, LDP, 1, C, sStage);
  #pragma unroll
    for (int i = 0; i < 4; ++i)
  #pragma unroll
      for (int j = 0; j < NJ; ++j) p.wX[ch * C * D + (ty + 16 * i) * D + tx + 16 * j] = acc[i][j];
    // Y = (gamma Q)^T dO
    for (int e = tid; e < C * D; e += PN) {
      const int at = (e / D) * LK + e % D;
      sQ[at] *= exp2f(sG[at]);
    }
    {
      float y[NJ][NJ];
      zero(y);
      mm_acc<NJ, NJ>(y, sQ, 1, LK, sBuf, LDP, 1, C, sStage);
  #pragma unroll
      for (int i = 0; i < NJ; ++i)
  #pragma unroll
        for (int j = 0; j < NJ; ++j) p.wY[ch * D * D + (ty + 16 * i) * D + tx + 16 * j] = y[i][j];
    }
  }

  // Khat = exp(G_last - G) K, Gam = exp(G_last); A and T for the gradient pass
  for (int e = tid; e < C * D; e += PN) {
    const int t = e / D, c = e % D;
    const float kh = sK[t * LK + c] * exp2f(sG[(C - 1) * LK + c] - sG[t * LK + c]);
    // the tensor-core state pass reads Khat as a tf32 operand, copied as it is
    p.wKh[ch * C * D + e] = kPrepTensorCores<D, TIn> ? tf32_round(kh) : kh;
  }
  if (tid < D) p.wGam[ch * D + tid] = exp2f(sG[(C - 1) * LK + tid]);
  for (int e = tid; e < C * C; e += PN) {
    p.wA[ch * C * C + e] = sA[(e / C) * LA + e % C];
    p.wT[ch * C * C + e] = sT[e];
  }
}

// ---------------------------------------------------------------------------
// bwd_state: the serial pass over chunk-end cotangents, last chunk first.  The
// recurrence acts on every value column of dS on its own (as the forward acts
// on the columns of S), so one CTA owns a 32-column slice of one chain.  The
// chunk's Khat and W tiles are copied to shared memory with cp.async one chunk
// ahead (two buffers), and the thread's X, Y and Gam entries of the next chunk are
// loaded into registers while the current chunk is computed, so the serial chain
// waits on no memory latency of its own operands.
// ---------------------------------------------------------------------------
constexpr int SC = 32;             // state columns per CTA
constexpr int ST_NTH = 16 * SC;    // threads (ty, tx): 16 x SC

// Shared layout: two buffers of the chunk's Khat and W tiles (as copied), the CTA's
// 32-column slice of dS held transposed (row stride LT, so a thread reads four
// consecutive k of its column as one float4 on distinct banks), and the dU slice.
template <int D>
struct StateLayout {
  static constexpr int LT = D + 4;
  static constexpr int oBuf = 0, BUF = 2 * C * D;  // Khat tile, then the W tile
  static constexpr int oS = oBuf + 2 * BUF, oU = oS + SC * LT;
  static constexpr int total = oU + C * SC;
  static constexpr size_t bytes = sizeof(float) * total;
};

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem) {
  const uint32_t a = (uint32_t)__cvta_generic_to_shared(smem);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(a), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
// wait until at most N of this thread's committed groups are still in flight
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <int D>
__global__ void __launch_bounds__(ST_NTH, 1) bwd_state_kernel(const BwdParams p) {
  using L = StateLayout<D>;
  constexpr int NSL = D / SC, MI = D / 16, LT = L::LT;
  static_assert(NSL >= 1 && D % SC == 0 && MI % 4 == 0, "state slices");
  extern __shared__ float4 smem_f4[];
  float *sm = reinterpret_cast<float *>(smem_f4);
  float *sdST = sm + L::oS, *sdU = sm + L::oU;
  const int tid = threadIdx.x, ty = tid / SC, tx = tid % SC;
  const int H = p.H;
  const int sl = blockIdx.x % NSL, rh = blockIdx.x / NSL;
  const int r = rh / H, h = rh % H;
  // the thread's state column; its dS rows are MI ty + i (side by side), its dU rows
  // ty + 16 i
  const int col = SC * sl + tx;
  const int jlo = p.cu_chunks[r], jhi = p.cu_chunks[r + 1];
  // copies chunk jc's Khat and W tiles into buffer b (one commit group)
  auto fetch = [&](int jc, int b) {
    const size_t ch = (size_t)jc * H + h;
    const float4 *gK = reinterpret_cast<const float4 *>(p.wKh + ch * C * D);
    const float4 *gW = reinterpret_cast<const float4 *>(p.wW + ch * C * D);
    float *dK = sm + L::oBuf + b * L::BUF, *dW = dK + C * D;
    for (int e = tid; e < C * D / 4; e += ST_NTH) {
      cp_async16(dK + 4 * e, gK + e);
      cp_async16(dW + 4 * e, gW + e);
    }
    cp_async_commit();
  };
  // the thread's X, Y and Gam entries of chunk jc
  float u[4], y[MI], gam[MI];
  auto load_own = [&](int jc, float *u_, float *y_, float *gam_) {
    const size_t ch = (size_t)jc * H + h;
#pragma unroll
    for (int i = 0; i < 4; ++i) u_[i] = p.wX[ch * C * D + (size_t)(ty + 16 * i) * D + col];
#pragma unroll
    for (int i = 0; i < MI; ++i) y_[i] = p.wY[ch * D * D + (size_t)(MI * ty + i) * D + col];
#pragma unroll
    for (int q = 0; q < MI / 4; ++q) {
      const float4 g4 = *reinterpret_cast<const float4 *>(p.wGam + ch * D + MI * ty + 4 * q);
      gam_[4 * q] = g4.x, gam_[4 * q + 1] = g4.y, gam_[4 * q + 2] = g4.z, gam_[4 * q + 3] = g4.w;
    }
  };
  if (jhi > jlo) {
    fetch(jhi - 1, 0);
    load_own(jhi - 1, u, y, gam);
  }
  const float *dfin = p.d_final ? p.d_final + ((size_t)r * H + h) * D * D : nullptr;
  float ds[MI];
#pragma unroll
  for (int i = 0; i < MI; ++i) ds[i] = dfin ? dfin[(size_t)(MI * ty + i) * D + col] : 0.f;
#pragma unroll
  for (int q = 0; q < MI / 4; ++q)
    *reinterpret_cast<float4 *>(sdST + tx * LT + MI * ty + 4 * q) =
        make_float4(ds[4 * q], ds[4 * q + 1], ds[4 * q + 2], ds[4 * q + 3]);
  for (int jc = jhi - 1, b = 0; jc >= jlo; --jc, b ^= 1) {
    const size_t ch = (size_t)jc * H + h;
    const bool more = jc > jlo;
    // the next chunk's tiles go to the other buffer, whose reads ended at the last
    // barrier of the previous chunk
    if (more) fetch(jc - 1, b ^ 1);
    if (more) cp_async_wait<1>(); else cp_async_wait<0>();
    __syncthreads();  // this chunk's tiles and the dS slice are complete
    const float *sKh = sm + L::oBuf + b * L::BUF, *sW = sKh + C * D;
    // dU = X + Khat dSn   (overwrites X)
#pragma unroll 2
    for (int k = 0; k < D; k += 4) {
      const float4 d4 = *reinterpret_cast<const float4 *>(sdST + tx * LT + k);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 kh = *reinterpret_cast<const float4 *>(sKh + (ty + 16 * i) * D + k);
        u[i] = fmaf(kh.x, d4.x, fmaf(kh.y, d4.y, fmaf(kh.z, d4.z, fmaf(kh.w, d4.w, u[i]))));
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      sdU[(ty + 16 * i) * SC + tx] = u[i];
      p.wX[ch * C * D + (size_t)(ty + 16 * i) * D + col] = u[i];
    }
    __syncthreads();
    // the next chunk's own entries, in flight while dS is formed
    float nu[4], ny[MI], ngam[MI];
    if (more) load_own(jc - 1, nu, ny, ngam);
    // dS = Diag(Gam) dSn + Y - W^T dU;  dSn overwrites Y for the gradient pass
    float acc[MI];
#pragma unroll
    for (int i = 0; i < MI; ++i) acc[i] = 0.f;
#pragma unroll 4
    for (int t = 0; t < C; ++t) {
      const float du = sdU[t * SC + tx];
#pragma unroll
      for (int q = 0; q < MI / 4; ++q) {
        const float4 w4 = *reinterpret_cast<const float4 *>(sW + t * D + MI * ty + 4 * q);
        acc[4 * q] = fmaf(w4.x, du, acc[4 * q]);
        acc[4 * q + 1] = fmaf(w4.y, du, acc[4 * q + 1]);
        acc[4 * q + 2] = fmaf(w4.z, du, acc[4 * q + 2]);
        acc[4 * q + 3] = fmaf(w4.w, du, acc[4 * q + 3]);
      }
    }
#pragma unroll
    for (int i = 0; i < MI; ++i) {
      p.wY[ch * D * D + (size_t)(MI * ty + i) * D + col] = ds[i];
      ds[i] = fmaf(gam[i], ds[i], y[i] - acc[i]);
    }
    __syncthreads();  // every read of sdST, sdU and this chunk's buffer is done
#pragma unroll
    for (int q = 0; q < MI / 4; ++q)
      *reinterpret_cast<float4 *>(sdST + tx * LT + MI * ty + 4 * q) =
          make_float4(ds[4 * q], ds[4 * q + 1], ds[4 * q + 2], ds[4 * q + 3]);
    if (more) {
#pragma unroll
      for (int i = 0; i < 4; ++i) u[i] = nu[i];
#pragma unroll
      for (int i = 0; i < MI; ++i) y[i] = ny[i], gam[i] = ngam[i];
    }
  }
  if (p.d_initial) {
    float *dst = p.d_initial + ((size_t)r * H + h) * D * D;
#pragma unroll
    for (int i = 0; i < MI; ++i) dst[(size_t)(MI * ty + i) * D + col] = ds[i];
  }
}

// ---------------------------------------------------------------------------
// bwd_state_tc (bf16 inputs, d = 128): the serial pass on the tensor cores.  One CTA
// per (request, head) holds dS^T in TMEM (lane = value column j, columns = key rows
// i) and takes the chunks last first:
//   dU^T = X^T + dSn^T Khat^T                 A = dSn^T (TMEM), B = Khat (rows = tokens)
//   dS^T = dSn^T Diag(Gam) + Y^T - dU^T W     A = dU^T (TMEM), B = W^T (rows = keys)
// The CUDA cores add X^T to the first product and write dU out, then write dSn out
// and form dSn^T Diag(Gam) + Y^T in place as the second product's accumulator.  Khat
// arrives tf32-rounded from the prep pass and is copied with cp.async two chunks
// ahead; W is transposed and rounded through registers one chunk ahead.  Products
// accumulate in fp32; their tf32 operands are the state (as TMEM holds it), dU
// (rounded to nearest), Khat and W.
// ---------------------------------------------------------------------------
constexpr int STC_NTH = 512;

struct StateTcLayout {
  static constexpr int D = 128;
  static constexpr int KB = C * D * 4;  // one Khat operand: 64 rows x 128 tf32 (32 KiB)
  static constexpr int WB = D * C * 4;  // one W^T operand: 128 rows x 64 tf32 (32 KiB)
  static constexpr int oK = 0, oW = 2 * KB, oGam = oW + 2 * WB;  // byte offsets
  static constexpr int oBar = oGam + 2 * D * 4;  // three mbarriers, then the TMEM address
  static constexpr size_t bytes = oBar + 32 + 1024;
};

__global__ void __launch_bounds__(STC_NTH, 1) bwd_state_tc_kernel(const BwdParams p) {
  using L = StateTcLayout;
  constexpr int D = L::D;
  constexpr uint32_t TS = 0, TU = 128;  // TMEM columns: dS^T, then dU^T
  extern __shared__ float4 smem_f4[];
  unsigned char *sb = align1024_shared(smem_f4);
  float *sGam = reinterpret_cast<float *>(sb + L::oGam);         // [2][128]
  uint64_t *bar = reinterpret_cast<uint64_t *>(sb + L::oBar);    // first, second, drain
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(sb + L::oBar + 24);
  const int tid = threadIdx.x, w = tid >> 5, ln = tid & 31;
  // warp w reaches TMEM lanes 32 (w % 4) .. + 31 (value columns j) and takes part w / 4
  // of the columns: tokens 16 part .. + 15 of dU^T, keys 32 part .. + 31 of dS^T
  const int qd = w & 3, part = w >> 2, j = 32 * qd + ln;
  const uint32_t lane = (uint32_t)(32 * qd) << 16;
  const int H = p.H, r = blockIdx.x / H, h = blockIdx.x % H;
  const int jlo = p.cu_chunks[r], jhi = p.cu_chunks[r + 1];
  if (w == 0) {
    tmem_alloc(s_tmem, 256);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(bar, 1);
    mbar_init(bar + 1, 1);
    mbar_init(bar + 2, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // Khat of chunk jc into operand buffer b (rows = tokens, K = keys); one commit group
  auto fetch_k = [&](int jc, int b) {
    const float4 *g = reinterpret_cast<const float4 *>(p.wKh + ((size_t)jc * H + h) * C * D);
    unsigned char *dst = sb + L::oK + b * L::KB;
#pragma unroll
    for (int q = 0; q < C * D / 4 / STC_NTH; ++q) {
      const int e = tid + q * STC_NTH, t = e >> 5, k = (e & 31) * 4;
      cp_async16(dst + sw128_chunk(C, t, k), g + e);
    }
    cp_async_commit();
  };
  // W of chunk jc, transposed (rows = keys, K = tokens): element e of the thread's four
  // takes key e % 128 and tokens 4 (e / 128) .. + 3 (a warp reads 128 bytes per token)
  float wv[4][4];
  auto load_w = [&](int jc) {
    const float *g = p.wW + ((size_t)jc * H + h) * C * D;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int e = tid + q * STC_NTH, i = e & (D - 1), t0 = (e >> 7) * 4;
#pragma unroll
      for (int u = 0; u < 4; ++u) wv[q][u] = g[(size_t)(t0 + u) * D + i];
    }
  };
  auto store_w = [&](int b) {
    unsigned char *dst = sb + L::oW + b * L::WB;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int e = tid + q * STC_NTH, i = e & (D - 1), t0 = (e >> 7) * 4;
      *reinterpret_cast<float4 *>(dst + sw128_chunk(D, i, t0)) =
          make_float4(tf32_round(wv[q][0]), tf32_round(wv[q][1]), tf32_round(wv[q][2]),
                      tf32_round(wv[q][3]));
    }
  };
  auto load_gam = [&](int jc, int b) {
    if (tid < D / 4)
      reinterpret_cast<float4 *>(sGam + b * D)[tid] =
          reinterpret_cast<const float4 *>(p.wGam + ((size_t)jc * H + h) * D)[tid];
  };

  const float *dfin = p.d_final ? p.d_final + ((size_t)r * H + h) * D * D : nullptr;
  float sv[32];
#pragma unroll
  for (int c = 0; c < 32; ++c) sv[c] = dfin ? dfin[(size_t)(32 * part + c) * D + j] : 0.f;
  if (jhi > jlo) {
    fetch_k(jhi - 1, 0);
    if (jhi - 1 > jlo) fetch_k(jhi - 2, 1);
    load_w(jhi - 1);
    load_gam(jhi - 1, 0);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = *s_tmem;
  tmem_st32(tm + lane + TS + 32 * part, sv);  // dS^T of the last chunk's end
  if (jhi > jlo) store_w(0);
  if (jhi - 1 > jlo) cp_async_wait<1>(); else cp_async_wait<0>();
  tmem_wait_st();
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  bool ok = true;
  uint32_t ph1 = 0, ph2 = 0;
  const uint32_t id64 = idesc_tf32(C), id128n = idesc_tf32(D, true);
  for (int jc = jhi - 1, b = 0; jc >= jlo; --jc, b ^= 1) {
    const size_t ch = (size_t)jc * H + h;
    if (tid == 0 && ok) {
      const uint32_t kb = smem_u32(sb + L::oK + b * L::KB);
#pragma unroll
      for (int s = 0; s < D / 8; ++s)
        mma_tf32_ts(tm + TU, tm + TS + 8 * s, sw128_desc(kb, C, s), id64, s > 0);
      mma_commit(bar);
    }
    // this chunk's X and Y entries, in flight under the first product
    float x[16], y[32];
#pragma unroll
    for (int tt = 0; tt < 16; ++tt) x[tt] = p.wX[ch * C * D + (size_t)(16 * part + tt) * D + j];
#pragma unroll
    for (int c = 0; c < 32; ++c) y[c] = p.wY[ch * D * D + (size_t)(32 * part + c) * D + j];
    ok = ok && mbar_wait(bar, ph1);
    ph1 ^= 1;
    tc_fence_after();
    // the first product is done with buffer b and with dSn^T
    if (jc - 2 >= jlo) fetch_k(jc - 2, b);
    if (jc - 1 >= jlo) {
      load_w(jc - 1);
      load_gam(jc - 1, b ^ 1);
    }
    if (ok) {
      float u[16];
      tmem_ld16(tm + lane + TU + 16 * part, u);
      tmem_wait_ld();
#pragma unroll
      for (int tt = 0; tt < 16; ++tt) {
        u[tt] += x[tt];
        p.wX[ch * C * D + (size_t)(16 * part + tt) * D + j] = u[tt];  // dU over X
        u[tt] = tf32_round(u[tt]);
      }
      tmem_st16(tm + lane + TU + 16 * part, u);
      tmem_ld32(tm + lane + TS + 32 * part, sv);
      tmem_wait_ld();
      const float *gam = sGam + b * D + 32 * part;
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        p.wY[ch * D * D + (size_t)(32 * part + c) * D + j] = sv[c];  // dSn over Y
        sv[c] = fmaf(gam[c], sv[c], y[c]);
      }
      tmem_st32(tm + lane + TS + 32 * part, sv);
    }
    if (jc - 1 >= jlo) store_w(b ^ 1);
    tmem_wait_st();
    if (jc - 2 >= jlo) cp_async_wait<1>(); else cp_async_wait<0>();  // Khat of jc - 1
    fence_async_smem();
    tc_fence_before();
    ok = __syncthreads_and(ok);
    tc_fence_after();
    if (!ok) break;
    if (tid == 0) {
      const uint32_t wb = smem_u32(sb + L::oW + b * L::WB);
#pragma unroll
      for (int s = 0; s < C / 8; ++s)
        mma_tf32_ts(tm + TS, tm + TU + 8 * s, sw128_desc(wb, D, s), id128n, true);
      mma_commit(bar + 1);
    }
    ok = mbar_wait(bar + 1, ph2);
    ph2 ^= 1;
    tc_fence_after();
  }
  cp_async_wait<0>();
  if (!__syncthreads_and(ok)) {
    if (tid == 0) {
      set_status(p.status, STATUS_TIMEOUT);
      mma_commit(bar + 2);  // covers every product issued
      mbar_wait(bar + 2, 0, 100000000ull);
    }
  } else if (p.d_initial) {
    tmem_ld32(tm + lane + TS + 32 * part, sv);
    tmem_wait_ld();
    float *dst = p.d_initial + ((size_t)r * H + h) * D * D;
#pragma unroll
    for (int c = 0; c < 32; ++c) dst[(size_t)(32 * part + c) * D + j] = sv[c];
  }
  tc_fence_before();
  __syncthreads();
  if (w == 0) {
    tc_fence_after();
    tmem_dealloc(tm, 256);
  }
}

// ---------------------------------------------------------------------------
// bwd_sprod (bf16 inputs, d = 128): the gradient pass's tile products on the tensor
// cores, in two stages per (chunk, head).  Each product has M = 128 TMEM lanes, its A
// operand in TMEM and its B operand K-major with the 128-byte swizzle in shared
// memory; tf32 operands rounded to nearest, fp32 accumulation.
// Stage 1, the products with the state (transposed, as in the forward):
//   U^T          = U~^T - S^T W^T    A = S^T (lane = value column), D starts as U~^T
//   d(gamma Q)^T = S dO^T            A = S (lane = key row)
//   dW^T         = -S dU^T           A = S
//   dKhat^T      = dSn U^T           A = dSn (lane = key row), B = U from the first product
// and dGam_i = sum_j dSn_ij S_ij (fp32 on the CUDA cores, from the unrounded values).
// Stage 2, the products of chunk-sized tiles, on lanes t = the chunk's 64 tokens (the
// other 64 lanes compute nothing anyone reads):
//   dP   = dO U^T                                 A = dO, B = U (rows s)
//   [T^T dU | T^T dW] = T^T [dU | dW]             A = T^T, B = [dU^T ; dW^T]
//                                                   (rows = 256 value columns, K = s)
//   dZ   = -[(T^T dU) U~^T + (T^T dW) W^T]        A = the product above (K = 256, read
//                                                   from TMEM as it stands), B = [U~ | W]
// U and dW stay on chip between the stages.  The results replace workspace tiles the
// gradient pass no longer reads: d(gamma Q) and dKhat over dSn, dGam over Gam, dP over
// T, dZ over U, T^T dU over dU, T^T dW over Khat.
// ---------------------------------------------------------------------------
constexpr int SP_NTH = 512;

struct SprodLayout {
  static constexpr int D = 128;
  // B operand tiles (byte offsets, 1024-byte aligned): U~ and W back to back (together
  // the K = 256 operand [U~ | W] of dZ), dO, dU and U (64 rows x 128 tf32 each), then
  // [dU^T ; dW^T] (256 rows x 64 tf32).  Before U and [dU^T ; dW^T] are written, their
  // space holds S (row stride LS floats, for both TMEM layouts of it) and, at its end,
  // the dGam partials.
  static constexpr int TILE = C * D * 4, LS = D + 4;
  static constexpr int oUt = 0, oW = TILE, oO = 2 * TILE, oDU = 3 * TILE, oU = 4 * TILE;
  static constexpr int oDUW = 5 * TILE, oS = oU, oPart = oDUW + 2 * TILE - 4 * D * 4;
  static_assert(oS + D * LS * 4 <= oPart, "S and the dGam partials overlap");
  static constexpr int oMisc = oDUW + 2 * TILE;  // four mbarriers, then the TMEM address
  static constexpr size_t bytes = oMisc + 48 + 1024;
};


__global__ void __launch_bounds__(SP_NTH, 1) bwd_sprod_kernel(const BwdParams p) {
  using L = SprodLayout;
  constexpr int D = L::D;
  // TMEM columns, stage 1: S^T, then dW^T | dKhat^T once the first product is done;
  // U~^T -> U^T; S; dSn; d(gamma Q)^T.  Stage 2: dO, then dZ; dP; T^T; [T^T dU | T^T dW].
  constexpr uint32_t TST = 0, TDW = 0, TDK = 64, TU = 128, TS = 192, TDS = 320, TGQ = 448;
  constexpr uint32_t TDO = 0, TZ = 0, TP = 128, TT = 192, TB = 256;
  extern __shared__ float4 smem_f4[];
  unsigned char *sb = align1024_shared(smem_f4);
  unsigned char *bUt = sb + L::oUt, *bW = sb + L::oW, *bO = sb + L::oO, *bDU = sb + L::oDU;
  unsigned char *bU = sb + L::oU, *bDUW = sb + L::oDUW;
  float *sPart = reinterpret_cast<float *>(sb + L::oPart);
  uint64_t *bar = reinterpret_cast<uint64_t *>(sb + L::oMisc);  // U^T, stage 1, 2a, 2b
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(sb + L::oMisc + 32);
  const int tid = threadIdx.x, w = tid >> 5, ln = tid & 31;
  const int H = p.H;
  const int jc = blockIdx.x / H, h = blockIdx.x % H;
  const int4 cd = p.chunks[jc];
  const int r = cd.x, cidx = cd.y, tok0 = cd.z, n = cd.w;
  const size_t ch = (size_t)jc * H + h;
  const float *S;
  if (cidx == 0)
    S = p.initial_state ? p.initial_state + ((size_t)r * H + h) * D * D : p.zero_state;
  else
    S = p.snaps + ((size_t)(p.cu_snap[r] + cidx - 1) * H + h) * D * D;
  const float *dSn = p.wY + ch * D * D;
  const float *Ut = p.wU + ch * C * D, *T = p.wT + ch * C * C;
  if (w == 0) {
    tmem_alloc(s_tmem, 512);
    tmem_relinquish();
  }
  if (tid == 0) {
#pragma unroll
    for (int i = 0; i < 4; ++i) mbar_init(bar + i, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }

  // B operands: U~, W, dO (rows past the chunk's end are zero) and dU, rows = tokens;
  // all of a thread's loads are issued before any of its stores
  {
    constexpr int NQ = C * D / 4 / SP_NTH;
    float4 utv[NQ], wv[NQ], uv[NQ], ov[NQ];
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
      const int e = tid + q * SP_NTH, t = e >> 5, k = (e & 31) * 4;
      utv[q] = *reinterpret_cast<const float4 *>(Ut + t * D + k);
      wv[q] = *reinterpret_cast<const float4 *>(p.wW + ch * C * D + t * D + k);
      uv[q] = *reinterpret_cast<const float4 *>(p.wX + ch * C * D + t * D + k);
      ov[q] = (p.d_o && t < n) ? *reinterpret_cast<const float4 *>(
                                     p.d_o + ((size_t)(tok0 + t) * H + h) * D + k)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
      const int e = tid + q * SP_NTH, t = e >> 5, k = (e & 31) * 4;
      *reinterpret_cast<float4 *>(bUt + sw128_chunk(C, t, k)) = tf32_round4(utv[q]);
      *reinterpret_cast<float4 *>(bW + sw128_chunk(C, t, k)) = tf32_round4(wv[q]);
      *reinterpret_cast<float4 *>(bDU + sw128_chunk(C, t, k)) = tf32_round4(uv[q]);
      *reinterpret_cast<float4 *>(bO + sw128_chunk(C, t, k)) = tf32_round4(ov[q]);
    }
  }
  // S into shared memory with whole-row loads: the TMEM layouts below read it by rows
  // (lane = key row) and by columns (lane = value column)
  float *sS = reinterpret_cast<float *>(sb + L::oS);
  {
    constexpr int NQ = D * D / 4 / SP_NTH;
    float4 sv4[NQ];
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
      const int e = tid + q * SP_NTH;
      sv4[q] = reinterpret_cast<const float4 *>(S + (size_t)(e >> 5) * D)[e & 31];
    }
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
      const int e = tid + q * SP_NTH;
      *reinterpret_cast<float4 *>(sS + (e >> 5) * L::LS + 4 * (e & 31)) = sv4[q];
    }
  }
  // warp w reaches TMEM lanes 32 (w % 4) .. + 31 and takes the 32-column part w / 4
  const int qd = w & 3, part = w >> 2, lrow = 32 * qd + ln;
  float4 dn[8];  // dSn row lrow, columns 32 part .. + 31, in flight across the barrier
  {
    const float4 *dr = reinterpret_cast<const float4 *>(dSn + (size_t)lrow * D + 32 * part);
#pragma unroll
    for (int q = 0; q < 8; ++q) dn[q] = dr[q];
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = *s_tmem;
  const uint32_t lane = (uint32_t)(32 * qd) << 16;
  {  // S^T: lane = value column, columns = key rows (consecutive lanes read one row)
    float v[32];
#pragma unroll
    for (int jj = 0; jj < 32; ++jj) v[jj] = tf32_round(sS[(32 * part + jj) * L::LS + lrow]);
    tmem_st32(tm + lane + TST + 32 * part, v);
  }
  {  // S and dSn: lane = key row, columns = value columns; the dGam partial sums
    float a[32], b[32];
    const float4 *sr = reinterpret_cast<const float4 *>(sS + lrow * L::LS + 32 * part);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      *reinterpret_cast<float4 *>(&a[4 * q]) = sr[q];
      *reinterpret_cast<float4 *>(&b[4 * q]) = dn[q];
    }
    float gs = 0.f;
#pragma unroll
    for (int jj = 0; jj < 32; ++jj) {
      gs = fmaf(a[jj], b[jj], gs);
      a[jj] = tf32_round(a[jj]);
      b[jj] = tf32_round(b[jj]);
    }
    sPart[part * D + lrow] = gs;
    tmem_st32(tm + lane + TS + 32 * part, a);
    tmem_st32(tm + lane + TDS + 32 * part, b);
  }
  {  // U~^T (the first product's accumulator, fp32): lane = value column, columns = tokens
    float v[16];
#pragma unroll
    for (int tt = 0; tt < 16; ++tt) v[tt] = Ut[(size_t)(16 * part + tt) * D + lrow];
    tmem_st16(tm + lane + TU + 16 * part, v);
  }
  tmem_wait_st();
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t id64 = idesc_tf32(64), id64n = idesc_tf32(64, true);
  if (tid == 0) {
    const uint32_t wb = smem_u32(bW), ob = smem_u32(bO);
#pragma unroll
    for (int s = 0; s < D / 8; ++s)
      mma_tf32_ts(tm + TU, tm + TST + 8 * s, sw128_desc(wb, C, s), id64n, true);
    mma_commit(bar);
#pragma unroll
    for (int s = 0; s < D / 8; ++s)
      mma_tf32_ts(tm + TGQ, tm + TS + 8 * s, sw128_desc(ob, C, s), id64, s > 0);
  }
  if (tid < D)  // dGam in a fixed order
    p.wGam[ch * D + tid] = (sPart[tid] + sPart[D + tid]) + (sPart[2 * D + tid] + sPart[3 * D + tid]);
  bool ok = mbar_wait(bar, 0);
  tc_fence_after();
  if (tid == 0 && ok) {  // S^T is consumed: dW^T = -S dU^T goes over its first half
    const uint32_t db = smem_u32(bDU);
#pragma unroll
    for (int s = 0; s < D / 8; ++s)
      mma_tf32_ts(tm + TDW, tm + TS + 8 * s, sw128_desc(db, C, s), id64n, s > 0);
  }
  if (ok) {  // U, rounded, to the B tile of dKhat^T and of dP
    float v[16];
    tmem_ld16(tm + lane + TU + 16 * part, v);
    tmem_wait_ld();
#pragma unroll
    for (int tt = 0; tt < 16; ++tt)
      *reinterpret_cast<float *>(bU + sw128_offset(C, 16 * part + tt, lrow)) = tf32_round(v[tt]);
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();  // also ends every read of the dGam partials
  tc_fence_after();
  if (tid == 0) {
    if (ok) {
      const uint32_t ub = smem_u32(bU);
#pragma unroll
      for (int s = 0; s < D / 8; ++s)
        mma_tf32_ts(tm + TDK, tm + TDS + 8 * s, sw128_desc(ub, C, s), id64, s > 0);
    }
    mma_commit(bar + 1);  // covers every product issued, whatever happened above
  }
  // dU^T rows of [dU^T ; dW^T] (rows = value columns c, K = tokens s) while it runs:
  // element e takes column e % 128 and tokens 4 (e / 128) .. + 3
#pragma unroll 1
  for (int q = 0; q < D * C / 4 / SP_NTH; ++q) {
    const int e = tid + q * SP_NTH, c = e & (D - 1), s0 = (e >> 7) * 4;
    const float *src = p.wX + ch * C * D + c;
    const float4 v = make_float4(src[(size_t)s0 * D], src[(size_t)(s0 + 1) * D],
                                 src[(size_t)(s0 + 2) * D], src[(size_t)(s0 + 3) * D]);
    *reinterpret_cast<float4 *>(bDUW + sw128_chunk(2 * D, c, s0)) = tf32_round4(v);
  }
  bool done = ok && mbar_wait(bar + 1, 0);
  tc_fence_after();
  if (done) {
    float v[16];
    tmem_ld16(tm + lane + TGQ + 16 * part, v);  // d(gamma Q)[token][key]
    tmem_wait_ld();
#pragma unroll
    for (int tt = 0; tt < 16; ++tt) p.wY[ch * D * D + (size_t)(16 * part + tt) * D + lrow] = v[tt];
    tmem_ld16(tm + lane + TDK + 16 * part, v);  // dKhat
    tmem_wait_ld();
#pragma unroll
    for (int tt = 0; tt < 16; ++tt)
      p.wY[ch * D * D + C * D + (size_t)(16 * part + tt) * D + lrow] = v[tt];
    tmem_ld16(tm + lane + TDW + 16 * part, v);  // dW^T: rows 128 + key of [dU^T ; dW^T]
    tmem_wait_ld();
#pragma unroll
    for (int q = 0; q < 4; ++q)  // 16-byte chunks; consecutive lanes on consecutive rows
      *reinterpret_cast<float4 *>(bDUW + sw128_chunk(2 * D, D + lrow, 16 * part + 4 * q)) =
          tf32_round4(make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]));
  }
  // stage 2: A operands on lanes t = 32 (w % 4) + lane for lane quarters 0 and 1; part
  // w / 4 takes a quarter of the columns
  const int t = lrow;
  fence_async_smem();
  tc_fence_before();
  done = __syncthreads_and(done);  // every stage-1 read of TMEM is done
  tc_fence_after();
  if (done && qd < 2) {
    float v[32];  // dO row t, value columns 32 part .. + 31, from its B tile (rounded)
#pragma unroll
    for (int q = 0; q < 8; ++q)
      *reinterpret_cast<float4 *>(&v[4 * q]) =
          *reinterpret_cast<const float4 *>(bO + sw128_chunk(C, t, 32 * part + 4 * q));
    tmem_st32(tm + lane + TDO + 32 * part, v);
    float tv[16];  // T^T row t: T[s][t] for s = 16 part .. + 15
#pragma unroll
    for (int ss = 0; ss < 16; ++ss) tv[ss] = tf32_round(T[(16 * part + ss) * C + t]);
    tmem_st16(tm + lane + TT + 16 * part, tv);
  }
  tmem_wait_st();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (tid == 0) {
    if (done) {
      const uint32_t ub = smem_u32(bU), dwb = smem_u32(bDUW), uwb = smem_u32(bUt);
#pragma unroll
      for (int s = 0; s < D / 8; ++s)
        mma_tf32_ts(tm + TP, tm + TDO + 8 * s, sw128_desc(ub, C, s), idesc_tf32(C), s > 0);
#pragma unroll
      for (int s = 0; s < C / 8; ++s)
        mma_tf32_ts(tm + TB, tm + TT + 8 * s, sw128_desc(dwb, 2 * D, s), idesc_tf32(2 * D),
                    s > 0);
      mma_commit(bar + 2);
      // the middle product is the next one's A, and dO's columns take dZ
      done = mbar_wait(bar + 2, 0);
      tc_fence_after();
      if (done) {
#pragma unroll
        for (int s = 0; s < 2 * D / 8; ++s)
          mma_tf32_ts(tm + TZ, tm + TB + 8 * s, sw128_desc(uwb, C, s), idesc_tf32(C, true),
                      s > 0);
      }
    }
    mma_commit(bar + 3);  // covers every product issued
  }
  done = __syncthreads_and(done) && mbar_wait(bar + 3, 0);
  if (!done && tid == 0) set_status(p.status, STATUS_TIMEOUT);
  tc_fence_after();
  // Results through shared memory (the B tiles are free once every product is done):
  // lane t writes its row segments, then the CTA stores whole rows to the workspace.
  // Row strides 1,040 and 272 bytes put a warp's 16-byte writes on distinct banks.
  constexpr int RB = 1040, RS = 272, oSP = 64 * RB, oSZ = oSP + 64 * RS;
  if (done && qd < 2) {
    float v[32];
    float4 *rb = reinterpret_cast<float4 *>(sb + t * RB);  // [T^T dU | T^T dW] row t
    float4 *rp = reinterpret_cast<float4 *>(sb + oSP + t * RS) + 4 * part;  // dP
    float4 *rz = reinterpret_cast<float4 *>(sb + oSZ + t * RS) + 4 * part;  // dZ
    tmem_ld16(tm + lane + TP + 16 * part, v);
    tmem_wait_ld();
#pragma unroll
    for (int q = 0; q < 4; ++q) rp[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    tmem_ld16(tm + lane + TZ + 16 * part, v);
    tmem_wait_ld();
#pragma unroll
    for (int q = 0; q < 4; ++q) rz[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {  // columns 64 part + 32 hh .. + 31
      tmem_ld32(tm + lane + TB + 64 * part + 32 * hh, v);
      tmem_wait_ld();
#pragma unroll
      for (int q = 0; q < 8; ++q)
        rb[16 * part + 8 * hh + q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    }
  }
  tc_fence_before();
  if (__syncthreads_and(done)) {
    // 6,144 float4: T^T dU over dU, T^T dW over Khat (64 rows x 64 float4), then dP over T
    // and dZ over U (64 rows x 16 float4 each); a warp stores 512 contiguous bytes
#pragma unroll 4
    for (int q = 0; q < 6144 / SP_NTH; ++q) {
      const int e = tid + q * SP_NTH;
      float4 x;
      float *dst;
      if (e < 4096) {
        const int row = e >> 6, c4 = e & 63;
        x = *reinterpret_cast<const float4 *>(sb + row * RB + 16 * c4);
        dst = (c4 < 32 ? p.wX : p.wKh) + ch * C * D + (size_t)row * D + 4 * (c4 & 31);
      } else {
        const int e2 = (e - 4096) & 1023, row = e2 >> 4, c4 = e2 & 15;
        const bool z = e >= 5120;
        x = *reinterpret_cast<const float4 *>(sb + (z ? oSZ : oSP) + row * RS + 16 * c4);
        dst = (z ? p.wU2 + ch * C * D : p.wT + ch * C * C) + (size_t)row * C + 4 * c4;
      }
      *reinterpret_cast<float4 *>(dst) = x;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (!done && tid == 0) mbar_wait(bar + 3, 0, 100000000ull);  // let issued products finish
  __syncthreads();
  if (w == 0) {
    tc_fence_after();
    tmem_dealloc(tm, 512);
  }
}

// ---------------------------------------------------------------------------
// bwd_grad: every token gradient of one chunk
// ---------------------------------------------------------------------------
template <int D>
struct GradLayout {
  static constexpr int oK = 0, oQ = oK + C * D, oV = oQ + C * D, oO = oV + C * D;
  static constexpr int oG = oO + C * D, oP = oG + C * D, oT = oP + C * C;
  static constexpr int oStage = oT + C * C, oB = oStage + stage_floats(C, D);
  static constexpr int oDb = oB + C, oX = oDb + C, oPart = oX + D, oGam = oPart + 16 * D;
  static constexpr int total = oGam + D;
  static constexpr size_t bytes = sizeof(float) * total;
};

template <int D, typename TIn>
__global__ void __launch_bounds__(grad_threads<D, TIn>(), 1) bwd_grad_kernel(const BwdParams p) {
  using L = GradLayout<D>;
  // every dense product comes from bwd_sprod (tensor cores) when it ran
  constexpr bool PRE = kPrepTensorCores<D, TIn>;
  // 16 x TX threads: thread (ty, tx) owns rows ty + 16 i and columns tx + TX j of a tile
  constexpr int TX = grad_threads<D, TIn>() / 16, GN = 16 * TX, NJ = D / TX, NC = C / TX;
  extern __shared__ float4 smem_f4[];
  float *sm = reinterpret_cast<float *>(smem_f4);
  float *sK = sm + L::oK, *sQ = sm + L::oQ, *sV = sm + L::oV, *sO = sm + L::oO;
  float *sG = sm + L::oG, *sP = sm + L::oP, *sT = sm + L::oT, *sStage = sm + L::oStage;
  float *sB = sm + L::oB, *sDb = sm + L::oDb, *sExtra = sm + L::oX, *sPart = sm + L::oPart;
  float *sGam = sm + L::oGam;
  const int tid = threadIdx.x, ty = tid / TX, tx = tid % TX;
  const int H = p.H;
  const int jc = blockIdx.x / H, h = blockIdx.x % H;
  const int4 cd = p.chunks[jc];
  const int r = cd.x, cidx = cd.y, tok0 = cd.z, n = cd.w;
  const size_t ch = (size_t)jc * H + h;
  const float *S;
  if (cidx == 0)
    S = p.initial_state ? p.initial_state + ((size_t)r * H + h) * D * D : p.zero_state;
  else
    S = p.snaps + ((size_t)(p.cu_snap[r] + cidx - 1) * H + h) * D * D;
  const float *dSn = p.wY + ch * D * D;
  const float *dU = p.wX + ch * C * D;
  const float *W = p.wW + ch * C * D;
  const float *Ut = p.wU + ch * C * D;
  float *U = p.wU2 + ch * C * D;

  if constexpr (PRE) {
    // bwd_sprod's d(gamma Q), dP and dZ tiles copied in while the rows stage: into the
    // O tile (dO is not staged here) and the P and T tiles they are folded into
    const float4 *gq = reinterpret_cast<const float4 *>(dSn);
    const float4 *gp = reinterpret_cast<const float4 *>(p.wT + ch * C * C);
    const float4 *gz = reinterpret_cast<const float4 *>(U);  // dZ over U, [C][C]
    for (int e = tid; e < C * D / 4; e += GN) cp_async16(sO + 4 * e, gq + e);
    for (int e = tid; e < C * C / 4; e += GN) {
      cp_async16(sP + 4 * e, gp + e);
      cp_async16(sT + 4 * e, gz + e);
    }
    cp_async_commit();
  }
  stage_rows<D, TIn, GN>(sK, D, static_cast<const TIn *>(p.k), tok0, n, H, h);
  stage_rows<D, TIn, GN>(sQ, D, static_cast<const TIn *>(p.q), tok0, n, H, h);
  stage_rows<D, TIn, GN>(sV, D, static_cast<const TIn *>(p.v), tok0, n, H, h);
  if constexpr (!PRE) stage_rows<D, float, GN>(sO, D, p.d_o, tok0, n, H, h);  // PRE: not read
  if (tid < C) sDb[tid] = 0.f;
  if constexpr (PRE) cp_async_wait<0>();  // made visible by stage_gate's barriers
  stage_gate<D, GN>(sG, sB, p, tok0, n, h);

  // the thread's elements: rows ty + 16 i, columns tx + TX j
  float accQ[4][NJ], accK[4][NJ], accG[4][NJ], acc[4][NJ];
  const float *G63 = sG + (C - 1) * D;

  // the thread's elements of a precomputed C x D product
  auto load_own = [&](const float *src) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < NJ; ++j) acc[i][j] = src[(ty + 16 * i) * D + tx + TX * j];
  };
  if constexpr (!PRE) {
    // U = U~ - W S  (U~ loaded before the product so its latency hides under it)
    float ut[4][NJ];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < NJ; ++j) ut[i][j] = Ut[(ty + 16 * i) * D + tx + TX * j];
    zero(acc);
    mm_acc<4, NJ>(acc, W, D, 1, S, D, 1, D, sStage);
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        const int e = (ty + 16 * i) * D + tx + TX * j;
        U[e] = ut[i][j] - acc[i][j];
      }
  }
  // d(gamma Q) = dO S^T  ->  dQ = d(gamma Q) gamma,  dG = d(gamma Q) gamma q
  if constexpr (PRE) {
    load_own(sO);  // bwd_sprod's d(gamma Q), copied into the O tile above
  } else {
    zero(acc);
    mm_acc<4, NJ>(acc, sO, D, 1, S, 1, D, D, sStage);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      const int e = (ty + 16 * i) * D + tx + TX * j;
      const float gq = acc[i][j] * exp2f(sG[e]);
      accQ[i][j] = gq;
      accG[i][j] = gq * sQ[e];
      accK[i][j] = 0.f;
    }
  // dP = tril(dO U^T)  (from bwd_sprod, over T, when it ran)
  {
    float pp[4][NC];
    if constexpr (PRE) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < NC; ++j) pp[i][j] = sP[(ty + 16 * i) * C + tx + TX * j];  // dP
    } else {
      zero(pp);
      mm_acc<4, NC>(pp, sO, D, 1, U, 1, D, D, sStage);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < NC; ++j) {
        const int t = ty + 16 * i, s = tx + TX * j;
        sP[t * C + s] = s <= t ? pp[i][j] : 0.f;
      }
  }
  // dKhat = U dSn^T  ->  dK += dKhat Gam/gamma,  dG -= dKhat Khat,  dG_last += sum_t dKhat Khat
  if constexpr (PRE) {
    load_own(dSn + C * D);  // and dKhat over its second half
  } else {
    zero(acc);
    mm_acc<4, NJ>(acc, U, D, 1, dSn, 1, D, D, sStage);
  }
#pragma unroll
  for (int j = 0; j < NJ; ++j) {
    float colsum = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int c = tx + TX * j, e = (ty + 16 * i) * D + c;
      const float f = exp2f(G63[c] - sG[e]);
      const float kh = sK[e] * f;
      accK[i][j] = fmaf(acc[i][j], f, accK[i][j]);
      accG[i][j] = fmaf(-acc[i][j], kh, accG[i][j]);
      colsum = fmaf(acc[i][j], kh, colsum);
    }
    sPart[ty * D + tx + TX * j] = colsum;
  }
  // dGam = rowsum(dSn * S): warp w takes rows w, w + 8, ...; lanes walk the row
  if constexpr (PRE) {
    if (tid < D) sGam[tid] = p.wGam[ch * D + tid];  // from bwd_sprod, over Gam
  } else {
    const int w = tid >> 5, ln = tid & 31;
#pragma unroll 4
    for (int row = w; row < D; row += GN / 32) {
      float a[D / 32], b[D / 32];
#pragma unroll
      for (int q = 0; q < D / 32; ++q) {
        a[q] = dSn[(size_t)row * D + ln + 32 * q];
        b[q] = S[(size_t)row * D + ln + 32 * q];
      }
      float v = 0.f;
#pragma unroll
      for (int q = 0; q < D / 32; ++q) v = fmaf(a[q], b[q], v);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
      if (ln == 0) sGam[row] = v;
    }
  }
  __syncthreads();
  // dG_last += dGam Gam + the partial column sums, in a fixed order (same on every run)
  if (tid < D) {
    float e = sGam[tid] * exp2f(G63[tid]);
    for (int y = 0; y < 16; ++y) e += sPart[y * D + tid];
    sExtra[tid] = e;
  }

  // dW = -dU S^T (into the dO tile; the sync above ends every read of that tile);
  // with the tensor cores, bwd_sprod has already taken every product with dW
  if constexpr (!PRE) {
    zero(acc);
    mm_acc<4, NJ>(acc, dU, D, 1, S, 1, D, D, sStage);
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < NJ; ++j) sO[(ty + 16 * i) * D + tx + TX * j] = -acc[i][j];
  }
  if constexpr (!PRE) {
    float4 tv[C * C / 4 / GN];
#pragma unroll
    for (int q = 0; q < C * C / 4 / GN; ++q)
      tv[q] = reinterpret_cast<const float4 *>(p.wT + ch * C * C)[tid + q * GN];
#pragma unroll
    for (int q = 0; q < C * C / 4 / GN; ++q)
      reinterpret_cast<float4 *>(sT)[tid + q * GN] = tv[q];
  }
  // T^T dU -> dV = Diag(beta) T^T dU, dbeta += (T^T dU) . v  (T^T dU from bwd_sprod, over
  // dU, when it ran)
  if constexpr (PRE) {
    load_own(dU);
  } else {
    zero(acc);
    mm_acc<4, NJ>(acc, sT, 1, C, dU, D, 1, C, sStage);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = ty + 16 * i;
    float rs = 0.f;
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      const int c = tx + TX * j;
      rs = fmaf(acc[i][j], sV[t * D + c], rs);
      if constexpr (!PRE) sV[t * D + c] = acc[i][j];  // T^T dU for dZ (own elements only)
      if (t < n) p.dv[((size_t)(tok0 + t) * H + h) * D + c] = sB[t] * acc[i][j];
    }
    rs = row_sum<TX>(rs);
    if (tx == 0) sDb[t] += rs;
  }
  // T^T dW -> d(gamma K) = Diag(beta) T^T dW;  dbeta += (T^T dW) . (gamma k)  (from
  // bwd_sprod, over dW, when it ran)
  if constexpr (PRE) {
    load_own(p.wKh + ch * C * D);
  } else {
    zero(acc);
    mm_acc<4, NJ>(acc, sT, 1, C, sO, D, 1, C, sStage);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = ty + 16 * i;
    float rs = 0.f;
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      const int e = t * D + tx + TX * j;
      const float gm = exp2f(sG[e]), kg = gm * sK[e];
      const float dkg = sB[t] * acc[i][j];
      accK[i][j] = fmaf(dkg, gm, accK[i][j]);
      accG[i][j] = fmaf(dkg, kg, accG[i][j]);
      rs = fmaf(acc[i][j], kg, rs);
      if constexpr (!PRE) sO[e] = acc[i][j];  // T^T dW for dZ (own elements only)
    }
    rs = row_sum<TX>(rs);
    if (tx == 0) sDb[t] += rs;
  }
  // dZ = -[(T^T dU) U~^T + (T^T dW) W^T];  dA = tril_strict(Diag(beta) dZ) into the T tile;
  // dbeta += sum_{s<t} dZ_ts A_ts
  {
    float av[4][NC];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < NC; ++j) av[i][j] = p.wA[ch * C * C + (ty + 16 * i) * C + tx + TX * j];
    float tt[4][NC];  // -dZ  (dZ from bwd_sprod, over U, when it ran)
    if constexpr (PRE) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < NC; ++j)
          tt[i][j] = -sT[(ty + 16 * i) * C + tx + TX * j];  // dZ, copied in above
    } else {
      zero(tt);
      mm_acc<4, NC>(tt, sV, D, 1, Ut, 1, D, D, sStage);
      mm_acc<4, NC>(tt, sO, D, 1, W, 1, D, D, sStage);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int t = ty + 16 * i;
      float rs = 0.f;
#pragma unroll
      for (int j = 0; j < NC; ++j) {
        const int s = tx + TX * j;
        const float dz = -tt[i][j];
        const bool low = s < t;
        if (low) rs = fmaf(dz, av[i][j], rs);
        sT[t * C + s] = low ? sB[t] * dz : 0.f;  // dA (T is no longer needed)
      }
      rs = row_sum<TX>(rs);
      if (tx == 0) sDb[t] += rs;
    }
  }

  if constexpr (PRE) {
    // Gated Gram cotangents on the tensor cores, one row block b at a time (reference
    // rows r0 = 16 b and r1 = r0 + 15, as below), transposed to M = 128 TMEM lanes, one
    // per channel c; tf32 operands rounded to nearest, fp32 accumulation:
    //   lower: [P1 | A1]^T[c][t] = sum_{s < r0 + 16} Kb^T[c][s] [dP ; dA][t][s],  t in block b
    //          Kb[s][c] = k_s e^{G_r0 - G_s}  (A, in TMEM);  B rows: 16 dP rows, 16 dA rows
    //   upper: O2^T[c][s] = sum_{t >= r0} (Q'^T[c][t] dP[t][s] + K'^T[c][t] dA[t][s]),
    //          s in block b;  Q'_t = q_t e^{G_t - G_r1}, K'_t = k_t e^{G_t - G_r1}
    // Terms past the triangles vanish (dP and dA are zero there; every factor is finite).
    // The CUDA cores scale the results by e^{G_t - G_r0} and e^{G_r1 - G_s} and hand them
    // to each element's owner through shared memory.
    constexpr uint32_t TLA = 0, TUA = 64, TLD = 192, TUD = 224;  // TMEM columns (of 256)
    unsigned char *bL = align1024_shared(sO);  // lower B: 32 rows x 64 K (8 KiB)
    unsigned char *bUp = bL + 8192;            // upper B: 16 rows x 128 K (8 KiB)
    float *x1 = sV, *x2 = sV + 16 * D, *x3 = sV + 32 * D;  // P1, A1, O2 scaled: [16][D]
    uint64_t *gbar = reinterpret_cast<uint64_t *>(sStage);  // sStage is unused here
    uint32_t *g_tmem = reinterpret_cast<uint32_t *>(sStage + 4);
    const int w = tid >> 5, ln = tid & 31, qd = w & 3, cg = w >> 2, c = 32 * qd + ln;
    const uint32_t lane = (uint32_t)(32 * qd) << 16;
    if (w == 0) {
      tmem_alloc(g_tmem, 256);
      tmem_relinquish();
    }
    if (tid == 0) {
      mbar_init(gbar, 1);
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = *g_tmem;
    bool ok = true;
#pragma unroll  // the owners' accumulators are indexed by b
    for (int b = 0; b < 4; ++b) {
      const int r0 = 16 * b, r1 = r0 + 15, KL = r0 + 16, KU = C - r0;
      // A operands: lane c, 8 columns per store; warp column group cg takes every 4th 8
      for (int s0 = 8 * cg; s0 < KL; s0 += 32) {
        float v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int s2 = s0 + u;
          v[u] = tf32_round(sK[s2 * D + c] * exp2f(sG[r0 * D + c] - sG[s2 * D + c]));
        }
        tmem_st8(tm + lane + TLA + s0, v);
      }
      for (int u0 = 8 * cg; u0 < 2 * KU; u0 += 32) {
        const bool kq = u0 >= KU;  // K' half (8-column groups never straddle KU)
        const float *src = kq ? sK : sQ;
        float v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int t = r0 + u0 + u - (kq ? KU : 0);
          v[u] = tf32_round(src[t * D + c] * exp2f(sG[t * D + c] - sG[r1 * D + c]));
        }
        tmem_st8(tm + lane + TUA + u0, v);
      }
      // B operands, one 16-byte chunk per step
      for (int e = tid; e < 32 * (KL / 4); e += GN) {  // rows n (dP, then dA), K = s
        const int nrow = e / (KL / 4), k0 = 4 * (e % (KL / 4));
        const float *row = (nrow < 16 ? sP : sT) + (r0 + (nrow & 15)) * C + k0;
        *reinterpret_cast<float4 *>(bL + sw128_chunk(32, nrow, k0)) =
            tf32_round4(*reinterpret_cast<const float4 *>(row));
      }
      for (int e = tid; e < 16 * (2 * KU / 4); e += GN) {  // rows n = s - r0, K = t' (dP, dA)
        const int nrow = e & 15, k0 = 4 * (e >> 4);
        const bool ka = k0 >= KU;
        const float *col = (ka ? sT : sP) + (r0 + k0 - (ka ? KU : 0)) * C + r0 + nrow;
        *reinterpret_cast<float4 *>(bUp + sw128_chunk(16, nrow, k0)) =
            tf32_round4(make_float4(col[0], col[C], col[2 * C], col[3 * C]));
      }
      tmem_wait_st();
      fence_async_smem();
      tc_fence_before();
      __syncthreads();
      tc_fence_after();
      if (tid == 0 && ok) {
        const uint32_t lb = smem_u32(bL), ub = smem_u32(bUp);
        for (int ks = 0; ks < KL / 8; ++ks)
          mma_tf32_ts(tm + TLD, tm + TLA + 8 * ks, sw128_desc(lb, 32, ks), idesc_tf32(32), ks > 0);
        for (int ks = 0; ks < 2 * KU / 8; ++ks)
          mma_tf32_ts(tm + TUD, tm + TUA + 8 * ks, sw128_desc(ub, 16, ks), idesc_tf32(16), ks > 0);
        mma_commit(gbar);
      }
      ok = ok && mbar_wait(gbar, (uint32_t)(b & 1));
      tc_fence_after();
      if (ok) {  // lane c: column group cg reads 8 of the 32 + 16 result columns
        float v[8];
        const int tb = 8 * (cg & 1);  // rows t (or s) tb .. tb + 7 of the block
        tmem_ld8(tm + lane + TLD + 8 * cg, v);  // P1 (cg 0, 1) or A1 (cg 2, 3)
        tmem_wait_ld();
        float *dst = cg < 2 ? x1 : x2;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int t = r0 + tb + u;
          dst[(tb + u) * D + c] = v[u] * exp2f(sG[t * D + c] - sG[r0 * D + c]);
        }
        if (cg < 2) {
          tmem_ld8(tm + lane + TUD + tb, v);  // O2
          tmem_wait_ld();
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int s2 = r0 + tb + u;
            x3[(tb + u) * D + c] = v[u] * exp2f(sG[r1 * D + c] - sG[s2 * D + c]);
          }
        }
      }
      tc_fence_before();
      ok = __syncthreads_and(ok);
      tc_fence_after();
      if (ok) {  // the element owners: row t = r0 + ty, columns tx + TX j
#pragma unroll
        for (int j = 0; j < NJ; ++j) {
          const int cc = tx + TX * j, e = ty * D + cc, et = (r0 + ty) * D + cc;
          const float p1 = x1[e], a1 = x2[e], o2 = x3[e];
          accQ[b][j] += p1;
          accK[b][j] += a1 + o2;
          accG[b][j] = fmaf(sQ[et], p1, fmaf(sK[et], a1 - o2, accG[b][j]));
        }
      }
      __syncthreads();  // x tiles, B tiles and TMEM are free for the next block
    }
    if (!ok && tid == 0) {
      set_status(p.status, STATUS_TIMEOUT);
      mma_commit(gbar);  // covers every product issued
      mbar_wait(gbar, 0, 100000000ull);
      mbar_wait(gbar, 1, 100000000ull);
    }
    tc_fence_before();
    __syncthreads();
    if (w == 0) {
      tc_fence_after();
      tmem_dealloc(tm, 256);
    }
  } else {
    // Gated Gram cotangents of P (dP in the P tile) and A (dA in the T tile), one row
    // block at a time, with the block factorisation of exp(G_t - G_s), t >= s:
    //   lower (row t of block b, reference r0 = 16 b):
    //     P1_t = sum_{s<=t} dP_ts k_s e^{G_t-G_s}  -> dq, dG += q P1
    //     A1_t = sum_{s<t}  dA_ts k_s e^{G_t-G_s}  -> dk, dG += k A1     (one k table)
    //   upper (row s of block b, reference r1 = 16 b + 15):
    //     P2_s + A2_s = sum_{t>=s} (dP_ts q_t + dA_ts k_t) e^{G_t-G_s}  -> dk, dG -= k (P2 + A2)
    // The dO and V tiles are dead here and hold the gate tables.
  #pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int r0 = 16 * b, r1 = r0 + 15;
      __syncthreads();
      if constexpr (NJ == 4) {  // one float4 chunk x (columns x + TX q) per step
        for (int e = tid; e < (r0 + 16) * TX; e += GN) {
          const int t = e / TX, x = e % TX;
          float v[4];
  #pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int c = x + TX * q;
            v[q] = sK[t * D + c] * exp2f(sG[r0 * D + c] - sG[t * D + c]);
          }
          *reinterpret_cast<float4 *>(sO + t * D + 4 * x) = make_float4(v[0], v[1], v[2], v[3]);
        }
      } else {
        for (int e = tid; e < (r0 + 16) * D; e += GN) {
          const int c = e % D;
          sO[e - c + gate_pos<TX, NJ>(c)] = sK[e] * exp2f(sG[r0 * D + c] - sG[e]);
        }
      }
      __syncthreads();
      {
        const int t = r0 + ty;
        float op[NJ], oa[NJ];
  #pragma unroll
        for (int j = 0; j < NJ; ++j) op[j] = oa[j] = 0.f;
  #pragma unroll 4
        for (int s2 = 0; s2 <= t; ++s2) {
          const float dp = sP[t * C + s2], da = sT[t * C + s2];
          float tb[NJ];
  #pragma unroll
          for (int q = 0; q < NJ / 4; ++q)
            *reinterpret_cast<float4 *>(&tb[4 * q]) =
                *reinterpret_cast<const float4 *>(sO + s2 * D + 4 * gate_chunk<TX, NJ>(tx, q));
  #pragma unroll
          for (int j = 0; j < NJ; ++j) {
            op[j] = fmaf(dp, tb[j], op[j]);
            oa[j] = fmaf(da, tb[j], oa[j]);
          }
        }
  #pragma unroll
        for (int j = 0; j < NJ; ++j) {
          const int c = tx + TX * j, e = t * D + c;
          const float f = exp2f(sG[e] - sG[r0 * D + c]);
          const float p1 = op[j] * f, a1 = oa[j] * f;
          accQ[b][j] += p1;
          accK[b][j] += a1;
          accG[b][j] = fmaf(sQ[e], p1, fmaf(sK[e], a1, accG[b][j]));
        }
      }
      __syncthreads();
      if constexpr (NJ == 4) {
        for (int e = r0 * TX + tid; e < C * TX; e += GN) {
          const int t = e / TX, x = e % TX;
          float qv[4], kv[4];
  #pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int c = x + TX * q;
            const float f = exp2f(sG[t * D + c] - sG[r1 * D + c]);
            qv[q] = sQ[t * D + c] * f;
            kv[q] = sK[t * D + c] * f;
          }
          *reinterpret_cast<float4 *>(sO + t * D + 4 * x) = make_float4(qv[0], qv[1], qv[2], qv[3]);
          *reinterpret_cast<float4 *>(sV + t * D + 4 * x) = make_float4(kv[0], kv[1], kv[2], kv[3]);
        }
      } else {
        for (int e = r0 * D + tid; e < C * D; e += GN) {
          const int c = e % D, at = e - c + gate_pos<TX, NJ>(c);
          const float f = exp2f(sG[e] - sG[r1 * D + c]);
          sO[at] = sQ[e] * f;
          sV[at] = sK[e] * f;
        }
      }
      __syncthreads();
      {
        const int s2 = r0 + ty;
        float o2[NJ];
  #pragma unroll
        for (int j = 0; j < NJ; ++j) o2[j] = 0.f;
  #pragma unroll 4
        for (int t = s2; t < C; ++t) {
          const float dp = sP[t * C + s2], da = sT[t * C + s2];
          float qb[NJ], kb[NJ];
  #pragma unroll
          for (int q = 0; q < NJ / 4; ++q) {
            *reinterpret_cast<float4 *>(&qb[4 * q]) =
                *reinterpret_cast<const float4 *>(sO + t * D + 4 * gate_chunk<TX, NJ>(tx, q));
            *reinterpret_cast<float4 *>(&kb[4 * q]) =
                *reinterpret_cast<const float4 *>(sV + t * D + 4 * gate_chunk<TX, NJ>(tx, q));
          }
  #pragma unroll
          for (int j = 0; j < NJ; ++j) o2[j] = fmaf(dp, qb[j], fmaf(da, kb[j], o2[j]));
        }
  #pragma unroll
        for (int j = 0; j < NJ; ++j) {
          const int c = tx + TX * j, e = s2 * D + c;
          const float v2 = o2[j] * exp2f(sG[r1 * D + c] - sG[e]);
          accK[b][j] += v2;
          accG[b][j] = fmaf(-sK[e], v2, accG[b][j]);
        }
      }
    }
  }

  // dg = reverse cumsum of dG (the last-row terms reach every row); write the gradients
  __syncthreads();
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      const int t = ty + 16 * i, c = tx + TX * j;
      sV[t * D + c] = accG[i][j];
      if (t < n) {
        const size_t o = ((size_t)(tok0 + t) * H + h) * D + c;
        p.dq[o] = accQ[i][j];
        p.dk[o] = accK[i][j];
      }
    }
  __syncthreads();
  if (tid < D) {  // dg = reverse cumulative sum of dG over the chunk, in place
    float run = sExtra[tid];
    for (int t = C - 1; t >= 0; --t) {
      run += sV[t * D + tid];
      sV[t * D + tid] = run;
    }
  }
  __syncthreads();
  // stored by the whole CTA; for gate logits x, times d log(alpha) / dx
  for (int e = tid; e < n * D; e += GN) {
    const size_t o = ((size_t)(tok0 + e / D) * H + h) * D + e % D;
    p.dg[o] = p.g_logits ? sV[e] * gate_logit_slope(__bfloat162float(p.g_logits[o])) : sV[e];
  }
  if (tid < C && tid < n) p.dbeta[(size_t)(tok0 + tid) * H + h] = sDb[tid];
}

template <typename K>
cudaError_t set_smem(K kernel, size_t bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <int D, typename TIn>
cudaError_t launch_bwd_d(const BwdParams &p, cudaStream_t stream) {
  cudaError_t e;
  const unsigned chunk_grid = (unsigned)((size_t)p.n_chunks * p.H);
  if (chunk_grid > 0) {
    if ((e = set_smem(bwd_prep_kernel<D, TIn>, PrepLayout<D>::bytes)) != cudaSuccess) return e;
    bwd_prep_kernel<D, TIn><<<chunk_grid, prep_threads<D, TIn>(), PrepLayout<D>::bytes, stream>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if constexpr (kPrepTensorCores<D, TIn>) {
    if ((e = set_smem(bwd_state_tc_kernel, StateTcLayout::bytes)) != cudaSuccess) return e;
    bwd_state_tc_kernel<<<(unsigned)(p.n_req * p.H), STC_NTH, StateTcLayout::bytes, stream>>>(p);
  } else {
    if ((e = set_smem(bwd_state_kernel<D>, StateLayout<D>::bytes)) != cudaSuccess) return e;
    bwd_state_kernel<D>
        <<<(unsigned)(p.n_req * p.H * (D / SC)), ST_NTH, StateLayout<D>::bytes, stream>>>(p);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if constexpr (kPrepTensorCores<D, TIn>) {
    if (chunk_grid > 0) {
      if ((e = set_smem(bwd_sprod_kernel, SprodLayout::bytes)) != cudaSuccess) return e;
      bwd_sprod_kernel<<<chunk_grid, SP_NTH, SprodLayout::bytes, stream>>>(p);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
  }
  if (chunk_grid > 0) {
    if ((e = set_smem(bwd_grad_kernel<D, TIn>, GradLayout<D>::bytes)) != cudaSuccess) return e;
    bwd_grad_kernel<D, TIn><<<chunk_grid, grad_threads<D, TIn>(), GradLayout<D>::bytes, stream>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace

// Workspace carve-up shared by the size query and the launch.
struct BwdWorkspace {
  size_t off_chunks, off_cu_chunks, off_cu_snap, off_snaps, off_zero;
  size_t off_A, off_T, off_W, off_U, off_Kh, off_X, off_Y, off_Gam, off_U2, total;
};

static size_t a256(size_t x) { return (x + 255) & ~size_t(255); }

BwdWorkspace backward_workspace(int n_req, int n_chunks, int n_snap, int H, int D) {
  BwdWorkspace w{};
  const size_t nch = (size_t)n_chunks * H, f = sizeof(float);
  size_t o = 0;
  auto take = [&](size_t bytes) { const size_t at = o; o = a256(o + bytes); return at; };
  w.off_chunks = take((size_t)n_chunks * sizeof(int4));
  w.off_cu_chunks = take((size_t)(n_req + 1) * sizeof(int32_t));
  w.off_cu_snap = take((size_t)(n_req + 1) * sizeof(int32_t));
  w.off_snaps = take((size_t)n_snap * H * D * D * f);
  w.off_zero = take((size_t)D * D * f);
  w.off_A = take(nch * C * C * f);
  w.off_T = take(nch * C * C * f);
  w.off_W = take(nch * C * D * f);
  w.off_U = take(nch * C * D * f);
  w.off_Kh = take(nch * C * D * f);
  w.off_X = take(nch * C * D * f);
  w.off_Y = take(nch * (size_t)D * D * f);
  w.off_Gam = take(nch * D * f);
  w.off_U2 = take(nch * C * D * f);
  w.total = o;
  return w;
}

cudaError_t launch_backward(const BackwardLaunch &b, cudaStream_t stream) {
  const BwdWorkspace w = backward_workspace(b.n_req, b.n_chunks, b.n_snap, b.H, b.D);
  char *ws = static_cast<char *>(b.workspace);
  BwdParams p{};
  p.q = b.q; p.k = b.k; p.v = b.v; p.g = b.g; p.beta = b.beta; p.g_logits = b.g_logits;
  p.initial_state = b.initial_state; p.d_o = b.d_o; p.d_final = b.d_final;
  p.dq = b.dq; p.dk = b.dk; p.dv = b.dv; p.dg = b.dg; p.dbeta = b.dbeta;
  p.d_initial = b.d_initial;
  p.chunks = reinterpret_cast<const int4 *>(ws + w.off_chunks);
  p.cu_chunks = reinterpret_cast<const int32_t *>(ws + w.off_cu_chunks);
  p.cu_snap = reinterpret_cast<const int32_t *>(ws + w.off_cu_snap);
  p.snaps = reinterpret_cast<const float *>(ws + w.off_snaps);
  p.zero_state = reinterpret_cast<const float *>(ws + w.off_zero);
  p.wA = reinterpret_cast<float *>(ws + w.off_A);
  p.wT = reinterpret_cast<float *>(ws + w.off_T);
  p.wW = reinterpret_cast<float *>(ws + w.off_W);
  p.wU = reinterpret_cast<float *>(ws + w.off_U);
  p.wKh = reinterpret_cast<float *>(ws + w.off_Kh);
  p.wX = reinterpret_cast<float *>(ws + w.off_X);
  p.wY = reinterpret_cast<float *>(ws + w.off_Y);
  p.wGam = reinterpret_cast<float *>(ws + w.off_Gam);
  p.wU2 = reinterpret_cast<float *>(ws + w.off_U2);
  p.n_req = b.n_req; p.n_chunks = b.n_chunks; p.H = b.H;
  p.status = device_status_word();
  if (b.D == 128)
    return b.in_dtype == KDA_BF16 ? launch_bwd_d<128, __nv_bfloat16>(p, stream)
                                  : launch_bwd_d<128, float>(p, stream);
  return b.in_dtype == KDA_BF16 ? launch_bwd_d<64, __nv_bfloat16>(p, stream)
                                : launch_bwd_d<64, float>(p, stream);
}

size_t backward_workspace_bytes(int n_req, int n_chunks, int n_snap, int H, int D) {
  return backward_workspace(n_req, n_chunks, n_snap, H, D).total;
}

void backward_offsets(int n_req, int n_chunks, int n_snap, int H, int D, size_t *chunks,
                      size_t *cu_chunks, size_t *cu_snap, size_t *snaps, size_t *zero) {
  const BwdWorkspace w = backward_workspace(n_req, n_chunks, n_snap, H, D);
  *chunks = w.off_chunks;
  *cu_chunks = w.off_cu_chunks;
  *cu_snap = w.off_cu_snap;
  *snaps = w.off_snaps;
  *zero = w.off_zero;
}

}  // namespace kda

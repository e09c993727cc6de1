// Chunked KDA prefill, SIMT fp32 kernel (sm_100a).
//
// Computes the chunk-parallel form of the KDA recurrence -- parallel inside a
// chunk of 64 tokens, serial between chunks ("Kimi K3 开源日来了", FlashKDA
// section) -- entirely in fp32 CUDA-core arithmetic.  It serves fp32 inputs
// (where the 1e-5 tolerance rules out tensor-core operand rounding), head
// dim 64, and the context-parallel local-state pass.
//
// Algebra of one chunk (state S0 at the chunk start, rows t = 0..63, G the
// chunk-local inclusive cumsum of g, gamma = exp(G)); derived by unrolling
// S_t = (I - b k k^T) Diag(alpha) S_{t-1} + b k v^T over the chunk:
//   A_ij = sum_c k_ic k_jc exp(G_ic - G_jc)   (j < i)
//   P_ij = sum_c q_ic k_jc exp(G_ic - G_jc)   (j <= i)
//   (I + Diag(b) A) [W | U~] = Diag(b) [gamma*K | V]        (forward substitution)
//   U  = U~ - W S0
//   O  = (gamma*Q) S0 + P U
//   S  = Diag(gamma_63) S0 + (exp(G_63 - G) * K)^T U
// The exponentials of A and P use 16-row blocks: for rows i of block a with
// first row r, exp(G_i - G_j) = exp(G_i - G_r) * exp(G_r - G_j).  The left
// factor is <= 1, the right factor is <= exp(5 * 15) because log alpha >= -5
// (the lower-bounded decay of KDA, CSDN post on the Kimi K3 technical report,
// section 一.1), so every factor is a finite, normal fp32 number.
//
// One CTA runs one (request, head, column slice) chain through all of its
// chunks; columns of the state are independent, so slicing dv is exact.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kThreads = 256;
constexpr int C = kChunk;  // 64

template <int DK, int DVS>
struct SimtLayout {
  static constexpr int XW = DK + DVS;  // row width of [W | U]
  static constexpr int oK = 0;
  static constexpr int oQ = oK + C * DK;
  static constexpr int oG = oQ + C * DK;
  static constexpr int oV = oG + C * DK;
  static constexpr int oA = oV + C * DVS;
  static constexpr int oP = oA + C * C;
  static constexpr int oX = oP + C * C;
  static constexpr int oS = oX + C * XW;
  static constexpr int oB = oS + DK * DVS;
  static constexpr int total = oB + C;
  static constexpr size_t bytes = sizeof(float) * total;
  static_assert(C * XW >= C * DK + 32 * DK, "scratch for the factor matrices must fit in X");
};

template <int DK, int DVS, typename TIn, typename TOut>
__global__ void __launch_bounds__(kThreads, 1) prefill_simt_kernel(const PrefillParams p) {
  using L = SimtLayout<DK, DVS>;
  constexpr int XW = L::XW;
  extern __shared__ float4 smem_f4[];
  float *smem = reinterpret_cast<float *>(smem_f4);
  float *sK = smem + L::oK, *sQ = smem + L::oQ, *sG = smem + L::oG, *sV = smem + L::oV;
  float *sA = smem + L::oA, *sP = smem + L::oP, *sX = smem + L::oX, *sS = smem + L::oS;
  float *sB = smem + L::oB;

  const int tid = threadIdx.x, lane = tid & 31;
  const int H = p.H, dv = p.dv;
  const int per_req = H * p.n_slices;
  const int pos = blockIdx.x / per_req, rem = blockIdx.x % per_req;
  const int r = p.order ? p.order[pos] : pos;
  const int h = rem / p.n_slices, slice = rem % p.n_slices;
  const int col0 = slice * DVS;
  const bool m_part = p.local_mode && col0 >= dv;  // transition columns
  const int bos = p.cu_seqlens[r], eos = p.cu_seqlens[r + 1];
  const int len = eos - bos;
  const TIn *gq = static_cast<const TIn *>(p.q);
  const TIn *gk = static_cast<const TIn *>(p.k);
  const TIn *gv = static_cast<const TIn *>(p.v);
  TOut *go = static_cast<TOut *>(p.o);
  // Offsets that would read or write outside the caller's buffers are
  // reported and skipped (uniform per CTA, before any barrier).
  if (bos < 0 || len < 0 || eos > p.total_tokens) {
    if (tid == 0) set_status(p.status, STATUS_BAD_SEQLENS);
    return;
  }
  bool snaps_ok = p.snapshot_stride > 0;
  if (snaps_ok && p.cu_snapshots[r + 1] - p.cu_snapshots[r] != len / p.snapshot_stride) {
    if (tid == 0) set_status(p.status, STATUS_BAD_SEQLENS);
    snaps_ok = false;
  }

  // ---- initial state of this column slice ---------------------------------
  for (int idx = tid; idx < DK * DVS; idx += kThreads) {
    const int i = idx / DVS, j = idx % DVS;
    float s = 0.f;
    if (p.local_mode) {
      if (m_part) s = (i == col0 - dv + j) ? 1.f : 0.f;
    } else if (p.initial_state) {
      s = p.initial_state[((size_t)(r * H + h) * DK + i) * dv + col0 + j];
    }
    sS[idx] = s;
  }

  // rows/cols owned by this thread in the 64 x DVS and DK x DVS products
  const int rg = tid / 16, cg = tid % 16;
  constexpr int JN = DVS / 16;

  for (int c0 = 0; c0 < len; c0 += C) {
    const int n = min(C, len - c0);
    __syncthreads();  // previous chunk fully consumed
    // ---- a1: load the chunk (padded rows are an exact no-op: k=q=g=b=v=0) --
    for (int idx = tid; idx < C * DK; idx += kThreads) {
      const int i = idx / DK, c = idx % DK;
      float kk = 0.f, qq = 0.f, gg = 0.f;
      if (i < n) {
        const size_t off = ((size_t)(bos + c0 + i) * H + h) * DK + c;
        kk = load_elem(gk, off);
        if (go) qq = load_elem(gq, off);
        if (p.g_logits) {
          gg = gate_from_logit(__bfloat162float(p.g_logits[off]));
        } else {
          gg = p.g[off];
          if (p.validate && !(gg >= kGateLower && gg <= 0.f)) set_status(p.status, STATUS_GATE_RANGE);
        }
      }
      sK[idx] = kk;
      sQ[idx] = qq;
      sG[idx] = gg;
    }
    for (int idx = tid; idx < C * DVS; idx += kThreads) {
      const int i = idx / DVS, j = idx % DVS;
      float vv = 0.f;
      if (i < n && !m_part) vv = load_elem(gv, ((size_t)(bos + c0 + i) * H + h) * dv + col0 + j);
      sV[idx] = vv;
    }
    if (tid < C) {
      float bb = 0.f;
      if (tid < n) {
        bb = p.beta[(size_t)(bos + c0 + tid) * H + h];
        if (p.validate && !(bb >= 0.f && bb <= 1.f)) set_status(p.status, STATUS_GATE_RANGE);
      }
      sB[tid] = bb;
    }
    __syncthreads();

    // ---- a2: chunk-local inclusive cumsum of the gate, per channel --------
    if (tid < DK) {
      float acc = 0.f;
      for (int i = 0; i < C; ++i) {
        acc += sG[i * DK + tid];
        sG[i * DK + tid] = acc;
      }
    }
    __syncthreads();

    // ---- a3: A and P by 16-row blocks with factorised exponentials --------
    for (int a = 0; a < C / 16; ++a) {
      const int r0 = 16 * a, nr = r0 + 16;
      float *sR = sX;               // [nr][DK]  k_j exp(G_r - G_j)
      float *sLk = sX + C * DK;     // [16][DK]  k_i exp(G_i - G_r)
      float *sLq = sLk + 16 * DK;   // [16][DK]  q_i exp(G_i - G_r)
      for (int idx = tid; idx < nr * DK; idx += kThreads) {
        const int j = idx / DK, c = idx % DK;
        sR[idx] = sK[idx] * expf(sG[r0 * DK + c] - sG[j * DK + c]);
      }
      for (int idx = tid; idx < 16 * DK; idx += kThreads) {
        const int i = r0 + idx / DK, c = idx % DK;
        const float e = expf(sG[i * DK + c] - sG[r0 * DK + c]);
        sLk[idx] = sK[i * DK + c] * e;
        sLq[idx] = sQ[i * DK + c] * e;
      }
      __syncthreads();
      for (int e = tid; e < 16 * C; e += kThreads) {
        const int il = e / C, j = e % C, i = r0 + il;
        float dA = 0.f, dP = 0.f;
        if (j <= i) {
          // rotate the channel index by lane so a warp hits distinct banks
          for (int cc = 0; cc < DK; ++cc) {
            const int c = (cc + lane) & (DK - 1);
            const float rj = sR[j * DK + c];
            dA = fmaf(sLk[il * DK + c], rj, dA);
            dP = fmaf(sLq[il * DK + c], rj, dP);
          }
        }
        sA[i * C + j] = (j < i) ? dA : 0.f;
        sP[i * C + j] = (j <= i) ? dP : 0.f;
      }
      __syncthreads();
    }

    // ---- a4: [W | U~] = (I + Diag(b) A)^-1 Diag(b) [gamma*K | V] ----------
    for (int idx = tid; idx < C * XW; idx += kThreads) {
      const int i = idx / XW, c = idx % XW;
      sX[idx] = (c < DK) ? sB[i] * expf(sG[i * DK + c]) * sK[i * DK + c]
                         : sB[i] * sV[i * DVS + (c - DK)];
    }
    __syncthreads();
    for (int col = tid; col < XW; col += kThreads) {
      for (int i = 1; i < C; ++i) {
        float acc = 0.f;
        for (int j = 0; j < i; ++j) acc = fmaf(sA[i * C + j], sX[j * XW + col], acc);
        sX[i * XW + col] -= sB[i] * acc;
      }
    }
    __syncthreads();

    // ---- a5: U = U~ - W S0 (in place in the right half of X) --------------
    {
      float acc[4][JN];
#pragma unroll
      for (int ii = 0; ii < 4; ++ii)
#pragma unroll
        for (int jj = 0; jj < JN; ++jj) acc[ii][jj] = 0.f;
      for (int c = 0; c < DK; ++c) {
        float av[4], bv[JN];
#pragma unroll
        for (int ii = 0; ii < 4; ++ii) av[ii] = sX[(rg + 16 * ii) * XW + c];
#pragma unroll
        for (int jj = 0; jj < JN; ++jj) bv[jj] = sS[c * DVS + cg + 16 * jj];
#pragma unroll
        for (int ii = 0; ii < 4; ++ii)
#pragma unroll
          for (int jj = 0; jj < JN; ++jj) acc[ii][jj] = fmaf(av[ii], bv[jj], acc[ii][jj]);
      }
#pragma unroll
      for (int ii = 0; ii < 4; ++ii)
#pragma unroll
        for (int jj = 0; jj < JN; ++jj)
          sX[(rg + 16 * ii) * XW + DK + cg + 16 * jj] -= acc[ii][jj];
    }
    // gate-scaled Q (for O) and K (for the state update), in place
    for (int idx = tid; idx < C * DK; idx += kThreads) {
      const int c = idx % DK;
      const float G = sG[idx];
      sQ[idx] *= expf(G);
      sK[idx] *= expf(sG[(C - 1) * DK + c] - G);
    }
    __syncthreads();

    // ---- a5/a6: O = (gamma*Q) S0 + P U, stored for the valid rows ---------
    if (go) {
      float acc[4][JN];
#pragma unroll
      for (int ii = 0; ii < 4; ++ii)
#pragma unroll
        for (int jj = 0; jj < JN; ++jj) acc[ii][jj] = 0.f;
      for (int c = 0; c < DK; ++c) {
        float av[4], bv[JN];
#pragma unroll
        for (int ii = 0; ii < 4; ++ii) av[ii] = sQ[(rg + 16 * ii) * DK + c];
#pragma unroll
        for (int jj = 0; jj < JN; ++jj) bv[jj] = sS[c * DVS + cg + 16 * jj];
#pragma unroll
        for (int ii = 0; ii < 4; ++ii)
#pragma unroll
          for (int jj = 0; jj < JN; ++jj) acc[ii][jj] = fmaf(av[ii], bv[jj], acc[ii][jj]);
      }
      for (int l = 0; l < C; ++l) {
        float av[4], bv[JN];
#pragma unroll
        for (int ii = 0; ii < 4; ++ii) av[ii] = sP[(rg + 16 * ii) * C + l];
#pragma unroll
        for (int jj = 0; jj < JN; ++jj) bv[jj] = sX[l * XW + DK + cg + 16 * jj];
#pragma unroll
        for (int ii = 0; ii < 4; ++ii)
#pragma unroll
          for (int jj = 0; jj < JN; ++jj) acc[ii][jj] = fmaf(av[ii], bv[jj], acc[ii][jj]);
      }
#pragma unroll
      for (int ii = 0; ii < 4; ++ii) {
        const int i = rg + 16 * ii;
        if (i < n) {
#pragma unroll
          for (int jj = 0; jj < JN; ++jj)
            store_elem(go, ((size_t)(bos + c0 + i) * H + h) * dv + col0 + cg + 16 * jj,
                       acc[ii][jj]);
        }
      }
    }
    __syncthreads();  // O read S0; the state update below overwrites it

    // ---- a5: S = Diag(gamma_63) S0 + Khat^T U -----------------------------
    {
      constexpr int CN = DK / 16;
      float acc[CN][JN];
#pragma unroll
      for (int cc = 0; cc < CN; ++cc)
#pragma unroll
        for (int jj = 0; jj < JN; ++jj) acc[cc][jj] = 0.f;
      for (int i = 0; i < C; ++i) {
        float av[CN], bv[JN];
#pragma unroll
        for (int cc = 0; cc < CN; ++cc) av[cc] = sK[i * DK + rg + 16 * cc];
#pragma unroll
        for (int jj = 0; jj < JN; ++jj) bv[jj] = sX[i * XW + DK + cg + 16 * jj];
#pragma unroll
        for (int cc = 0; cc < CN; ++cc)
#pragma unroll
          for (int jj = 0; jj < JN; ++jj) acc[cc][jj] = fmaf(av[cc], bv[jj], acc[cc][jj]);
      }
#pragma unroll
      for (int cc = 0; cc < CN; ++cc) {
        const int c = rg + 16 * cc;
        const float decay = expf(sG[(C - 1) * DK + c]);
#pragma unroll
        for (int jj = 0; jj < JN; ++jj) {
          float *s = &sS[c * DVS + cg + 16 * jj];
          *s = fmaf(decay, *s, acc[cc][jj]);
        }
      }
    }
    __syncthreads();

    // ---- a6: snapshot at request-local positions that are multiples of the stride
    if (snaps_ok && n == C && (c0 + C) % p.snapshot_stride == 0) {
      const size_t row = (size_t)p.cu_snapshots[r] + (c0 + C) / p.snapshot_stride - 1;
      float *dst = p.snapshots + (row * H + h) * (size_t)DK * dv;
      for (int idx = tid; idx < DK * DVS; idx += kThreads) {
        const int i = idx / DVS, j = idx % DVS;
        dst[(size_t)i * dv + col0 + j] = sS[idx];
      }
    }
  }
  __syncthreads();

  // ---- final state ----------------------------------------------------------
  if (p.local_mode) {
    for (int idx = tid; idx < DK * DVS; idx += kThreads) {
      const int i = idx / DVS, j = idx % DVS;
      if (m_part)
        p.m[((size_t)(r * H + h) * DK + i) * DK + (col0 - dv) + j] = sS[idx];
      else
        p.s_loc[((size_t)(r * H + h) * DK + i) * dv + col0 + j] = sS[idx];
    }
  } else if (p.final_state) {
    for (int idx = tid; idx < DK * DVS; idx += kThreads) {
      const int i = idx / DVS, j = idx % DVS;
      p.final_state[((size_t)(r * H + h) * DK + i) * dv + col0 + j] = sS[idx];
    }
  }
}

template <int DK, int DVS, typename TIn, typename TOut>
cudaError_t launch_typed(const PrefillParams &p, cudaStream_t stream) {
  using L = SimtLayout<DK, DVS>;
  auto kern = prefill_simt_kernel<DK, DVS, TIn, TOut>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)L::bytes);
  if (e != cudaSuccess) return e;
  const long long blocks = (long long)p.n_req * p.H * p.n_slices;
  if (blocks == 0) return cudaSuccess;
  kern<<<(unsigned)blocks, kThreads, L::bytes, stream>>>(p);
  return cudaGetLastError();
}

template <int DK, int DVS, typename TIn>
cudaError_t launch_out(const PrefillParams &p, kda_dtype out_dtype, cudaStream_t stream) {
  if (out_dtype == KDA_BF16) return launch_typed<DK, DVS, TIn, __nv_bfloat16>(p, stream);
  return launch_typed<DK, DVS, TIn, float>(p, stream);
}

}  // namespace

int prefill_simt_slices(int dk, int dv, bool local_mode) {
  const int cols = local_mode ? dv + dk : dv;
  return cols / 64;  // DVS = 64 for both head dims
}

cudaError_t launch_prefill_simt(const PrefillParams &p, kda_dtype in_dtype, kda_dtype out_dtype,
                                cudaStream_t stream) {
  if (p.dk == 128) {
    if (in_dtype == KDA_BF16) return launch_out<128, 64, __nv_bfloat16>(p, out_dtype, stream);
    return launch_out<128, 64, float>(p, out_dtype, stream);
  }
  if (in_dtype == KDA_BF16) return launch_out<64, 64, __nv_bfloat16>(p, out_dtype, stream);
  return launch_out<64, 64, float>(p, out_dtype, stream);
}

}  // namespace kda

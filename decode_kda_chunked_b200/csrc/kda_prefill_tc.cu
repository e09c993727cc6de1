// Chunked KDA prefill on the sm_100a tensor cores: TMA tile loads, tcgen05
// tf32 MMAs with fp32 accumulators in tensor memory (TMEM), fp32 SIMT for the
// cumulative gate, the exponentials and the triangular solve.
//
// The chunk algebra is that of the chunk-parallel form (tokens of a chunk in
// parallel, state passed between chunks in order: "Kimi K3 开源日来了",
// FlashKDA section), written transposed so that every MMA has M = 128 with
// one TMEM lane per feature channel (S^T, U^T, O^T have lanes = value
// channels, columns = key channels or tokens):
//
//   A | P   [128 x 16] per 16-column block b:  [L_b ; Lq_b] R_b^T           (A from TMEM)
//   W^T     = (gamma*K)^T (T Diag(b))^T                                      (A from TMEM)
//   U~^T    = V^T (T Diag(b))^T                                              (A from TMEM)
//   U^T     = U~^T - S^T W^T                                                 (A = S^T in TMEM)
//   O^T     = S^T (gamma*Q)^T + U^T P^T                                      (A = S^T, U^T in TMEM)
//   S^T    <- S^T Diag(gamma_63) + U^T Khat                                  (A = U^T in TMEM)
//
// Gate factorisation for A and P: for the 16-token column block b with last
// row r_b, exp(G_i - G_j) = exp(G_i - G_rb) * exp(G_rb - G_j).  The right
// factor is <= 1 for j <= r_b; the left factor is <= exp(5 * 15) for rows i
// of block b and <= 1 below it, and rows above block b (masked anyway) are
// set to zero.  Because log alpha >= -5 (the lower-bounded decay of KDA, CSDN
// post on the Kimi K3 technical report, section 一.1) every factor is a
// finite fp32 number.  Row i's left factors for earlier blocks follow from
// its own block's factor times the per-channel block-to-block decays
// exp(G_ra - G_rb), so each row needs one exponential per channel.
//
// All tensor-core operands are tf32 (B operands K-major with the 128-byte
// swizzle in shared memory): bf16 operands for the gate-scaled products would
// cost about 2e-3 of relative accuracy, tf32 stays near 5e-4.
//
// One CTA (4 warps) runs one (request, head) chain: 128 threads, TMEM lane =
// thread.  Thread 0 issues TMA loads and MMAs; every wait is bounded and a
// timeout is reported through the status word.
#include "kda_internal.cuh"
#include "kda_sm100.cuh"

namespace kda {
namespace {

using namespace sm100;

constexpr int C = 64;     // chunk
constexpr int DH = 128;   // head dim (dk = dv)
constexpr int NT = 128;   // threads per CTA

// ---- shared memory map (byte offsets from a 1024-aligned base) ----
constexpr uint32_t OFF_KRAW = 0;        // bf16 [64 x 128]: 2 TMA boxes of 64 cols (SW128)
constexpr uint32_t OFF_QRAW = 16384;
constexpr uint32_t OFF_VRAW = 32768;
constexpr uint32_t OFF_GRAW = 49152;    // fp32 [64 x 128]: 4 TMA boxes of 32 cols (SW128)
constexpr uint32_t RAW_BYTES = 81920;
constexpr uint32_t OFF_R = 81920;       // 4 x [16 x 128] tf32 B operands; later W [64 x 128]
constexpr uint32_t OFF_GQ = 114688;     // (gamma*Q) [64 x 128] tf32 B operand
constexpr uint32_t OFF_KHT = 147456;    // Khat^T [128 x 64] tf32 B operand
constexpr uint32_t OFF_TB = 180224;     // T Diag(beta) [64 x 64] tf32 B operand
constexpr uint32_t OFF_P = 196608;      // P [64 x 64] tf32 B operand
constexpr uint32_t OFF_E = 212992;      // E[b*4+a][128] = exp(G_ra - G_rb), b <= a (8 KB)
constexpr uint32_t OFF_EGR = 221184;    // exp(G_rb)[4][128] (2 KB)
constexpr uint32_t OFF_BETA = 223232;   // beta[64]
constexpr uint32_t OFF_BAR = 223488;    // mbarriers + TMEM base + flags
constexpr uint32_t SMEM_BYTES = 223616;
constexpr uint32_t SMEM_ALLOC = SMEM_BYTES + 1024;  // alignment slack
// T-solve scratch lives in the raw-tile region once the raw tiles are consumed.
constexpr uint32_t OFF_MS = 0;          // beta*A strict lower, fp32 [64][65]
constexpr uint32_t OFF_TI = 16640;      // T = (I + beta A)^-1, fp32 [64][65]
constexpr uint32_t OFF_Y = 33280;       // level products, fp32 [3][16][17]
constexpr int LD = 65;

// ---- TMEM column map (512 columns x 128 lanes of fp32) ----
constexpr uint32_t TM_S = 0;     // S^T (lane = value channel, col = key channel)
constexpr uint32_t TM_L = 128;   // A-operand scratch: L_b; later V^T [0,64) and (gK)^T [64,128)
constexpr uint32_t TM_AP = 256;  // A (lanes 0..63) and P (lanes 64..127), col = j
constexpr uint32_t TM_X1 = 320;  // W^T, later O^T
constexpr uint32_t TM_X2 = 384;  // U~^T -> U^T
constexpr uint32_t TM_COLS = 512;

struct TcMaps {
  CUtensorMap q, k, v, g;
};

__device__ __forceinline__ float bf16_at(const unsigned char *tile, int t, int c) {
  // bf16 [64 x 128] as two 64-column SW128 boxes
  const uint32_t off = (uint32_t)(c >> 6) * 8192u + (uint32_t)t * 128u +
                       ((uint32_t)(((c & 63) >> 3) ^ (t & 7)) << 4) + (uint32_t)(c & 7) * 2u;
  return __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(tile + off));
}
__device__ __forceinline__ uint32_t g_off(int t, int c) {
  // fp32 [64 x 128] as four 32-column SW128 boxes
  return (uint32_t)(c >> 5) * 8192u + (uint32_t)t * 128u +
         ((uint32_t)(((c & 31) >> 2) ^ (t & 7)) << 4) + (uint32_t)(c & 3) * 4u;
}
__device__ __forceinline__ float tf32_rna(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}

template <typename TOut>
__global__ void __launch_bounds__(NT, 1)
    prefill_tc_kernel(const PrefillParams p, const __grid_constant__ TcMaps maps) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char *sm = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float *sE = reinterpret_cast<float *>(sm + OFF_E);
  float *sEgr = reinterpret_cast<float *>(sm + OFF_EGR);
  float *sB = reinterpret_cast<float *>(sm + OFF_BETA);
  uint64_t *bar_tma = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
  uint64_t *bar_mma = bar_tma + 1;
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(bar_tma + 2);
  int *s_abort = reinterpret_cast<int *>(s_tmem + 1);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int H = p.H;
  const int r = p.order ? p.order[blockIdx.x / H] : blockIdx.x / H;
  const int h = blockIdx.x % H;
  const int bos = p.cu_seqlens[r], eos = p.cu_seqlens[r + 1];
  const int len = eos - bos;
  if (bos < 0 || len < 0 || eos > p.total_tokens) {  // uniform per CTA, before any barrier
    if (tid == 0) set_status(p.status, STATUS_BAD_SEQLENS);
    return;
  }
  bool snaps_ok = p.snapshot_stride > 0;
  if (snaps_ok && p.cu_snapshots[r + 1] - p.cu_snapshots[r] != len / p.snapshot_stride) {
    if (tid == 0) set_status(p.status, STATUS_BAD_SEQLENS);
    snaps_ok = false;
  }
  TOut *go = static_cast<TOut *>(p.o);

  if (warp == 0) tmem_alloc(s_tmem, TM_COLS);
  if (tid == 0) {
    mbar_init(bar_tma, 1);
    mbar_init(bar_mma, 1);
    *s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    tma_prefetch_desc(&maps.q);
    tma_prefetch_desc(&maps.k);
    tma_prefetch_desc(&maps.v);
    tma_prefetch_desc(&maps.g);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = *s_tmem;
  const uint32_t lane = (uint32_t)(warp * 32) << 16;  // this warp's TMEM lane quarter

  uint32_t tma_phase = 0, mma_phase = 0;
  auto issue_tma = [&](int c0) {
    mbar_expect_tx(bar_tma, RAW_BYTES);
    const int y = bos + c0;
    for (int half = 0; half < 2; ++half) {
      const int x = h * DH + 64 * half;
      tma_load_2d(sm + OFF_KRAW + 8192 * half, &maps.k, x, y, bar_tma);
      tma_load_2d(sm + OFF_QRAW + 8192 * half, &maps.q, x, y, bar_tma);
      tma_load_2d(sm + OFF_VRAW + 8192 * half, &maps.v, x, y, bar_tma);
    }
    for (int qd = 0; qd < 4; ++qd)
      tma_load_2d(sm + OFF_GRAW + 8192 * qd, &maps.g, h * DH + 32 * qd, y, bar_tma);
  };
  // thread 0 waits on an mbarrier, then the CTA synchronises; a timeout aborts the CTA
  auto wait_bar = [&](uint64_t *bar, uint32_t &phase) -> bool {
    if (tid == 0) {
      if (!mbar_wait(bar, phase)) {
        *s_abort = 1;
        set_status(p.status, STATUS_TIMEOUT);
      }
    }
    phase ^= 1u;
    __syncthreads();
    tc_fence_after();
    return *s_abort == 0;
  };
  auto commit_and_wait = [&]() -> bool {
    if (tid == 0) mma_commit(bar_mma);
    return wait_bar(bar_mma, mma_phase);
  };

  if (tid == 0 && len > 0) issue_tma(0);

  // ---- initial state -> S^T in TMEM (lane v holds S[:, v]) ----
  {
    const float *s0 = p.initial_state ? p.initial_state + ((size_t)(r * H + h)) * DH * DH : nullptr;
    for (int q = 0; q < 4; ++q) {
      float v[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = s0 ? s0[(size_t)(32 * q + j) * DH + tid] : 0.f;
      tmem_st32(tm + lane + TM_S + 32 * q, v);
    }
    tmem_wait_st();
  }

  bool ok = true;
  for (int c0 = 0; c0 < len && ok; c0 += C) {
    const int n = min(C, len - c0);
    if (tid < C) {
      float b = 0.f;
      if (tid < n) {
        b = p.beta[(size_t)(bos + c0 + tid) * H + h];
        if (p.validate && !(b >= 0.f && b <= 1.f)) set_status(p.status, STATUS_GATE_RANGE);
      }
      sB[tid] = b;
    }
    if (!(ok = wait_bar(bar_tma, tma_phase))) break;

    // ---- a2: cumulative gate (thread = channel), block-end tables -------------
    {
      const int c = tid;
      float acc = 0.f, gr[4];
#pragma unroll 8
      for (int t = 0; t < C; ++t) {
        float *gp = reinterpret_cast<float *>(sm + OFF_GRAW + g_off(t, c));
        float gv = 0.f;
        if (t < n) {
          gv = *gp;
          if (p.validate && !(gv >= kGateLower && gv <= 0.f)) set_status(p.status, STATUS_GATE_RANGE);
        }
        acc += gv;
        *gp = acc;
        if ((t & 15) == 15) gr[t >> 4] = acc;
      }
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        sEgr[b * DH + c] = __expf(gr[b]);
#pragma unroll
        for (int a = 0; a < 4; ++a)
          if (a >= b) sE[(b * 4 + a) * DH + c] = __expf(gr[a] - gr[b]);
      }
    }
    __syncthreads();

    // ---- a3 operands (thread = row): own-block factors, R_b, Khat^T, gamma*Q ----
    const bool kside = tid < C;
    const int i = tid & (C - 1);
    const int bi = i >> 4;
    const bool valid = i < n;
    float Lst[DH];
    {
      const unsigned char *xraw = sm + (kside ? OFF_KRAW : OFF_QRAW);
      const int rb = 16 * bi + 15;
#pragma unroll
      for (int c = 0; c < DH; c += 4) {
        const float4 gi = *reinterpret_cast<const float4 *>(sm + OFF_GRAW + g_off(i, c));
        const float4 grb = *reinterpret_cast<const float4 *>(sm + OFF_GRAW + g_off(rb, c));
        float x[4], f[4];
        const float giv[4] = {gi.x, gi.y, gi.z, gi.w}, grv[4] = {grb.x, grb.y, grb.z, grb.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          x[e] = valid ? bf16_at(xraw, i, c + e) : 0.f;
          f[e] = __expf(giv[e] - grv[e]);
          Lst[c + e] = x[e] * f[e];
        }
        if (kside) {
          // R_b row (i % 16) of block bi: k_i exp(G_rb - G_i); Khat = R * exp(G_63 - G_rb)
          float rv[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) rv[e] = tf32_rna(x[e] * __expf(grv[e] - giv[e]));
          *reinterpret_cast<float4 *>(sm + OFF_R + bi * 8192 + sw128_chunk(16, i & 15, c)) =
              make_float4(rv[0], rv[1], rv[2], rv[3]);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float kh = x[e] * __expf(grv[e] - giv[e]) * sE[(bi * 4 + 3) * DH + c + e];
            *reinterpret_cast<float *>(sm + OFF_KHT + sw128_offset(DH, c + e, i)) = tf32_rna(kh);
          }
        } else {
          float gq[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) gq[e] = tf32_rna(Lst[c + e] * sEgr[bi * DH + c + e]);
          *reinterpret_cast<float4 *>(sm + OFF_GQ + sw128_chunk(C, i, c)) =
              make_float4(gq[0], gq[1], gq[2], gq[3]);
        }
      }
    }
    fence_async_smem();

    // ---- a3: A and P, one 16-column block at a time -------------------------
    for (int b = 0; b < 4 && ok; ++b) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int c = 32 * q + j;
          v[j] = (b <= bi) ? tf32_rna(Lst[c] * sE[(b * 4 + bi) * DH + c]) : 0.f;
        }
        tmem_st32(tm + lane + TM_L + 32 * q, v);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncthreads();
      if (tid == 0) {
        tc_fence_after();
        const uint32_t id = idesc_tf32(16);
        const uint32_t rb = smem_u32(sm + OFF_R + b * 8192);
#pragma unroll 1
        for (int s = 0; s < DH / 8; ++s)
          mma_tf32_ts(tm + TM_AP + 16 * b, tm + TM_L + 8 * s, sw128_desc(rb, 16, s), id, s > 0);
      }
      ok = commit_and_wait();
    }
    if (!ok) break;

    // ---- V^T and (gamma*K)^T into TMEM (thread = channel) -------------------
    {
      const int c = tid;
      float v[32];
      for (int q = 0; q < 2; ++q) {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int t = 32 * q + j;
          v[j] = (t < n) ? tf32_rna(bf16_at(sm + OFF_VRAW, t, c)) : 0.f;
        }
        tmem_st32(tm + lane + TM_L + 32 * q, v);
      }
      for (int q = 0; q < 2; ++q) {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int t = 32 * q + j;
          const float G = *reinterpret_cast<const float *>(sm + OFF_GRAW + g_off(t, c));
          v[j] = (t < n) ? tf32_rna(bf16_at(sm + OFF_KRAW, t, c) * __expf(G)) : 0.f;
        }
        tmem_st32(tm + lane + TM_L + 64 + 32 * q, v);
      }
      tmem_wait_st();
    }
    __syncthreads();  // raw tiles consumed: the region becomes T-solve scratch

    // ---- a4: T = (I + Diag(beta) A)^-1 (blocked, fp32), P operand ------------
    float *Ms = reinterpret_cast<float *>(sm + OFF_MS);
    float *Ti = reinterpret_cast<float *>(sm + OFF_TI);
    float *Ys = reinterpret_cast<float *>(sm + OFF_Y);
    {
      float a[64];
      tmem_ld32(tm + lane + TM_AP, a);
      tmem_ld32(tm + lane + TM_AP + 32, a + 32);
      tmem_wait_ld();
      if (kside) {
        const float bi_ = sB[i];
#pragma unroll
        for (int j = 0; j < 64; ++j) Ms[i * LD + j] = (j < i) ? bi_ * a[j] : 0.f;
      } else {
#pragma unroll
        for (int j = 0; j < 64; j += 4)
          *reinterpret_cast<float4 *>(sm + OFF_P + sw128_chunk(C, i, j)) =
              make_float4(j + 0 <= i ? tf32_rna(a[j]) : 0.f, j + 1 <= i ? tf32_rna(a[j + 1]) : 0.f,
                          j + 2 <= i ? tf32_rna(a[j + 2]) : 0.f,
                          j + 3 <= i ? tf32_rna(a[j + 3]) : 0.f);
      }
    }
    __syncthreads();
    if (tid < C) {  // diagonal 16x16 blocks by forward substitution, one column per thread
      const int blk = tid >> 4, jj = tid & 15, o = 16 * blk;
      float x[16];
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        float acc = (k == jj) ? 1.f : 0.f;
#pragma unroll
        for (int l = 0; l < 16; ++l)
          if (l < k && l >= jj) acc -= Ms[(o + k) * LD + o + l] * x[l];
        x[k] = (k < jj) ? 0.f : acc;
        Ti[(o + k) * LD + o + jj] = x[k];
      }
    }
    __syncthreads();
    for (int d = 1; d < 4; ++d) {  // off-diagonal blocks, level by level
      const int nblk = 4 - d;
      for (int e = tid; e < nblk * 256; e += NT) {  // Y = sum_c Ms_{a,c} T_{c,b}
        const int bb = e >> 8, k = (e >> 4) & 15, j = e & 15, a = bb + d;
        float acc = 0.f;
        for (int cb = bb; cb < a; ++cb)
#pragma unroll
          for (int l = 0; l < 16; ++l)
            acc += Ms[(16 * a + k) * LD + 16 * cb + l] * Ti[(16 * cb + l) * LD + 16 * bb + j];
        Ys[(bb * 16 + k) * 17 + j] = acc;
      }
      __syncthreads();
      for (int e = tid; e < nblk * 256; e += NT) {  // T_ab = -T_aa Y
        const int bb = e >> 8, k = (e >> 4) & 15, j = e & 15, a = bb + d;
        float acc = 0.f;
#pragma unroll
        for (int l = 0; l < 16; ++l)
          acc += Ti[(16 * a + k) * LD + 16 * a + l] * Ys[(bb * 16 + l) * 17 + j];
        Ti[(16 * a + k) * LD + 16 * bb + j] = -acc;
      }
      __syncthreads();
    }
    if (kside) {  // TB = T Diag(beta), row i
#pragma unroll
      for (int j = 0; j < 64; j += 4) {
        float v4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          v4[e] = (j + e <= i) ? tf32_rna(Ti[i * LD + j + e] * sB[j + e]) : 0.f;
        *reinterpret_cast<float4 *>(sm + OFF_TB + sw128_chunk(C, i, j)) =
            make_float4(v4[0], v4[1], v4[2], v4[3]);
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && c0 + C < len) issue_tma(c0 + C);  // prefetch the next chunk

    // ---- a4: U~^T = V^T TB^T, W^T = (gK)^T TB^T ------------------------------
    if (tid == 0) {
      tc_fence_after();
      const uint32_t id = idesc_tf32(64);
      const uint32_t tb = smem_u32(sm + OFF_TB);
#pragma unroll 1
      for (int s = 0; s < C / 8; ++s) {
        mma_tf32_ts(tm + TM_X2, tm + TM_L + 8 * s, sw128_desc(tb, C, s), id, s > 0);
        mma_tf32_ts(tm + TM_X1, tm + TM_L + 64 + 8 * s, sw128_desc(tb, C, s), id, s > 0);
      }
    }
    if (!(ok = commit_and_wait())) break;

    // ---- W operand (rows = tokens, K = key channels) from W^T ---------------
    {
      float w[64];
      tmem_ld32(tm + lane + TM_X1, w);
      tmem_ld32(tm + lane + TM_X1 + 32, w + 32);
      tmem_wait_ld();
#pragma unroll
      for (int t = 0; t < C; ++t)
        *reinterpret_cast<float *>(sm + OFF_R + sw128_offset(C, t, tid)) = tf32_rna(w[t]);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---- a5: U^T = U~^T - S^T W^T ; O^T = S^T (gamma Q)^T ---------------------
    if (tid == 0) {
      tc_fence_after();
      const uint32_t idn = idesc_tf32(64, true), id = idesc_tf32(64);
      const uint32_t wb = smem_u32(sm + OFF_R), qb = smem_u32(sm + OFF_GQ);
#pragma unroll 1
      for (int s = 0; s < DH / 8; ++s) {
        mma_tf32_ts(tm + TM_X2, tm + TM_S + 8 * s, sw128_desc(wb, C, s), idn, true);
        mma_tf32_ts(tm + TM_X1, tm + TM_S + 8 * s, sw128_desc(qb, C, s), id, s > 0);
      }
    }
    if (!(ok = commit_and_wait())) break;

    // ---- S^T <- S^T Diag(gamma_63): column c scaled by exp(G_63,c) -----------
    for (int q = 0; q < 4; ++q) {
      float v[32];
      tmem_ld32(tm + lane + TM_S + 32 * q, v);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] *= sEgr[3 * DH + 32 * q + j];
      tmem_st32(tm + lane + TM_S + 32 * q, v);
    }
    tmem_wait_st();
    tc_fence_before();
    __syncthreads();

    // ---- a5: O^T += U^T P^T ; S^T += U^T Khat --------------------------------
    if (tid == 0) {
      tc_fence_after();
      const uint32_t id64 = idesc_tf32(64), id128 = idesc_tf32(128);
      const uint32_t pb = smem_u32(sm + OFF_P), kb = smem_u32(sm + OFF_KHT);
#pragma unroll 1
      for (int s = 0; s < C / 8; ++s) {
        mma_tf32_ts(tm + TM_X1, tm + TM_X2 + 8 * s, sw128_desc(pb, C, s), id64, true);
        mma_tf32_ts(tm + TM_S, tm + TM_X2 + 8 * s, sw128_desc(kb, DH, s), id128, true);
      }
    }
    if (!(ok = commit_and_wait())) break;

    // ---- a6: outputs (lane = value channel) and snapshots --------------------
    if (go) {
      float o[64];
      tmem_ld32(tm + lane + TM_X1, o);
      tmem_ld32(tm + lane + TM_X1 + 32, o + 32);
      tmem_wait_ld();
#pragma unroll
      for (int t = 0; t < C; ++t)
        if (t < n) store_elem(go, ((size_t)(bos + c0 + t) * H + h) * DH + tid, o[t]);
    }
    if (snaps_ok && n == C && (c0 + C) % p.snapshot_stride == 0) {
      const size_t row = (size_t)p.cu_snapshots[r] + (c0 + C) / p.snapshot_stride - 1;
      float *dst = p.snapshots + (row * H + h) * (size_t)DH * DH;
      for (int q = 0; q < 4; ++q) {
        float v[32];
        tmem_ld32(tm + lane + TM_S + 32 * q, v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) dst[(size_t)(32 * q + j) * DH + tid] = v[j];
      }
    }
    tc_fence_before();
    __syncthreads();
  }

  if (ok && p.final_state) {
    float *dst = p.final_state + ((size_t)(r * H + h)) * DH * DH;
    tc_fence_after();
    for (int q = 0; q < 4; ++q) {
      float v[32];
      tmem_ld32(tm + lane + TM_S + 32 * q, v);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 32; ++j) dst[(size_t)(32 * q + j) * DH + tid] = v[j];
    }
  }
  if (!ok && tid == 0) {
    // give in-flight copies and MMAs a bounded chance to land before TMEM is freed
    mbar_wait(bar_tma, tma_phase, 100000000ull);
    mbar_wait(bar_mma, mma_phase, 100000000ull);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_relinquish();
    tmem_dealloc(tm, TM_COLS);
  }
}

bool encode_map(CUtensorMap *m, const void *ptr, CUtensorMapDataType dt, uint64_t esize,
                uint64_t inner, uint64_t rows, uint32_t box_inner) {
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * esize};
  cuuint32_t box[2] = {box_inner, 64};
  cuuint32_t es[2] = {1, 1};
  return cuTensorMapEncodeTiled(m, dt, 2, const_cast<void *>(ptr), dims, strides, box, es,
                                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool prefill_tc_supported(int dk, int dv, kda_dtype in_dtype) {
  return dk == DH && dv == DH && in_dtype == KDA_BF16;
}

cudaError_t launch_prefill_tc(const PrefillParams &p, kda_dtype in_dtype, kda_dtype out_dtype,
                              cudaStream_t stream) {
  (void)in_dtype;
  if (p.n_req == 0) return cudaSuccess;
  TcMaps maps;
  const uint64_t T = (uint64_t)p.total_tokens, W = (uint64_t)p.H * DH;
  if (!encode_map(&maps.q, p.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, W, T, 64) ||
      !encode_map(&maps.k, p.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, W, T, 64) ||
      !encode_map(&maps.v, p.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, W, T, 64) ||
      !encode_map(&maps.g, p.g, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, W, T, 32))
    return cudaErrorInvalidValue;
  cudaError_t e;
  if (out_dtype == KDA_BF16) {
    e = cudaFuncSetAttribute(prefill_tc_kernel<__nv_bfloat16>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    prefill_tc_kernel<__nv_bfloat16><<<(unsigned)(p.n_req * p.H), NT, SMEM_ALLOC, stream>>>(p, maps);
  } else {
    e = cudaFuncSetAttribute(prefill_tc_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    prefill_tc_kernel<float><<<(unsigned)(p.n_req * p.H), NT, SMEM_ALLOC, stream>>>(p, maps);
  }
  return cudaGetLastError();
}

}  // namespace kda

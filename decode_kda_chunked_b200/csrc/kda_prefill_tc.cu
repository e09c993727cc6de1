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
//   A | P   [128 x 32(b+1)] per 32-row block b: [L ; Lq] R'_b^T             (A from TMEM)
//   Y^T     = V^T - S^T (gamma*K)^T                                          (A = S^T in TMEM)
//   U^T     = Y^T (T Diag(b))^T                                              (A = Y^T in TMEM)
//   O^T     = S^T (gamma*Q)^T + U^T P^T                                      (A = S^T, U^T in TMEM)
//   S^T    <- S^T Diag(gamma_63) + U^T Khat                                  (A = U^T in TMEM)
// U = T Diag(b) (V - (gamma*K) S) is the chunk form's U~ - W S with W never formed:
// Y needs only the state and the chunk's inputs, so it runs while the workers solve T.
//
// Gate factorisation for A and P: rows come in two 32-row blocks b with reference
// rows m_b = 32 b + 15, and exp(G_i - G_j) = exp(G_i - G_mb) * exp(G_mb - G_j) for a
// row i of block b and a column j <= i.  The left factor is <= exp(5 * 15) (rows
// i < m_b) or <= 1; the right factor is <= exp(5 * 16) (columns j > m_b) or <= 1.
// Because log alpha >= -5 (the lower-bounded decay of KDA, CSDN post on the Kimi K3
// technical report, section 一.1) every factor is a finite fp32 number, and only
// masked products (j > i) can overflow; they are dropped by selection, never
// multiplied.  Column j's right factor for block b follows from its own block's
// factor times the block-to-block decay exp(G_mb - G_m(j)) <= 1, so each row
// needs one exponential per channel.  Each block's product runs as two 8-step
// accumulation chains over the halves of the key channels, summed on read-out.
//
// All tensor-core operands are tf32 (B operands K-major with the 128-byte
// swizzle in shared memory): bf16 operands for the gate-scaled products would
// cost about 2e-3 of relative accuracy, tf32 stays near 5e-4.
//
// One CTA runs one (request, head) chain with 16 worker warps and one control
// warp.  Worker warp w reaches the TMEM lane quarter w % 4, and the four warps
// sharing a quarter split the columns.  The control warp issues the TMA loads
// and every tcgen05.mma; workers and control hand off through mbarriers
// (operands ready / MMA done / raw tiles consumed), so MMA issue never stalls
// a worker warp.  Every wait is bounded; a timeout is reported through the
// status word.
#include "kda_internal.cuh"
#include "kda_sm100.cuh"

namespace kda {
namespace {

using namespace sm100;

constexpr int C = 64;     // chunk
constexpr int DH = 128;   // head dim (dk = dv)
constexpr int NT = 512;   // worker threads per CTA: 16 warps (plus one control warp)
constexpr float LOG2E = 1.4426950408889634f;

// Thread (g, l): warp w = tid / 32 owns TMEM lane quarter w % 4, so
// l = 32 (w % 4) + tid % 32 is the thread's TMEM lane, and g = w / 4 picks a
// quarter of the columns (32 of 128, or 16 of 64).

// ---- shared memory map (byte offsets from a 1024-aligned base) ----
constexpr uint32_t OFF_KRAW = 0;        // bf16 [64 x 128]: 2 TMA boxes of 64 cols (SW128)
constexpr uint32_t OFF_QRAW = 16384;
constexpr uint32_t OFF_VRAW = 32768;
constexpr uint32_t OFF_GRAW = 49152;    // fp32 [64 x 128]: 4 TMA boxes of 32 cols (SW128), or
                                        // bf16 gate logits in its first half (2 boxes of 64
                                        // cols, as q/k/v); rewritten in place with
                                        // log2(e) * cumsum(g)
constexpr uint32_t RAW_BYTES = 81920;
// Once every raw tile is read, the raw region holds the B operands R'_b of
// the A|P products: row block b (32 rows) has 32(b+1) rows at byte 16384 b.
__host__ __device__ constexpr uint32_t rp_off(int b) { return 16384u * b; }
constexpr uint32_t OFF_R = 81920;       // R scratch [64 x 132] fp32, then T-solve scratch
constexpr int LDT = 65;                 // padded row stride of the T-solve scratch
constexpr int LDR = 132;                // padded row stride of the fp32 R scratch [64][132]
constexpr uint32_t OFF_MS = OFF_R;                  // beta*A strict lower
constexpr uint32_t OFF_TI = OFF_R + 64 * LDT * 4;   // T = (I + beta A)^-1
constexpr uint32_t OFF_GQ = 115712;     // (gamma*Q) [64 x 128] tf32 B operand; once the O^T
                                        // product has read it, (gamma*K) [64 x 128]
constexpr uint32_t OFF_KHT = 148480;    // Khat^T [128 x 64] tf32 B operand
constexpr uint32_t OFF_TB = 181248;     // T Diag(beta) [64 x 64] tf32 B operand
constexpr uint32_t OFF_P = 197632;      // P [64 x 64] tf32 B operand
constexpr uint32_t OFF_Y = 214016;      // the T-solve products ([2][16][17], then [32][33])
constexpr uint32_t OFF_EGR = 222208;    // exp(G_rb)[4][128], r_b = 16 b + 15
constexpr uint32_t OFF_SEG = 224256;    // cumsum segment totals [4][128]
constexpr uint32_t OFF_GR2 = 226304;    // log2(e) * G at rows 16 b + 15 [4][128]
constexpr uint32_t OFF_BETA = 228352;   // beta[64]
constexpr uint32_t OFF_BAR = 228608;    // mbarriers + TMEM base + flags
constexpr uint32_t SMEM_BYTES = 228704;
static_assert(OFF_TI + 64 * LDT * 4 <= OFF_GQ, "T-solve scratch must fit the R region");
static_assert(OFF_R + 64 * LDR * 4 <= OFF_GQ, "R scratch must fit the R region");
constexpr uint32_t SMEM_ALLOC = SMEM_BYTES + 1024;  // alignment slack

// ---- TMEM column map (512 columns x 128 lanes of fp32) ----
constexpr uint32_t TM_S = 0;     // S^T (lane = value channel, col = key channel)
constexpr uint32_t TM_L = 128;   // L* (A operand of A|P); later V^T -> Y^T in [0,64)
// A (lanes 0..63) | P (lanes 64..127) of the rows of 32-row block b: 32(b+1) columns,
// summed over two halves of the key channels held apart (two accumulators each)
constexpr uint32_t TM_AP = 256;  // up to column 448
__host__ __device__ constexpr uint32_t ap_col(int b, int half) {
  return TM_AP + (b == 0 ? 32u * half : 64u + 64u * half);
}
constexpr uint32_t TM_X2 = 320;  // U^T (alias A|P once the solve has read it)
constexpr uint32_t TM_O = 448;   // O^T (own columns: issued right after the A|P products)
constexpr uint32_t TM_COLS = 512;

struct TcMaps {
  CUtensorMap q, k, v, g;
};

__device__ __forceinline__ uint32_t bf16_off(int t, int c) {
  // bf16 [64 x 128] as two 64-column SW128 boxes
  return (uint32_t)(c >> 6) * 8192u + (uint32_t)t * 128u +
         ((uint32_t)(((c & 63) >> 3) ^ (t & 7)) << 4) + (uint32_t)(c & 7) * 2u;
}
__device__ __forceinline__ float bf16_at(const unsigned char *tile, int t, int c) {
  return __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(tile + bf16_off(t, c)));
}
// four consecutive channels c..c+3 (c % 4 == 0) of row t
__device__ __forceinline__ void bf16_x4(const unsigned char *tile, int t, int c, float *x) {
  const uint2 u = *reinterpret_cast<const uint2 *>(tile + bf16_off(t, c));
  x[0] = __uint_as_float(u.x << 16);
  x[1] = __uint_as_float(u.x & 0xFFFF0000u);
  x[2] = __uint_as_float(u.y << 16);
  x[3] = __uint_as_float(u.y & 0xFFFF0000u);
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
// [64 x 65] fp32 scratch: the padded stride puts a warp's row walk and column
// walk on 32 distinct banks and keeps addresses affine in the loop indices.
__device__ __forceinline__ int rot(int r, int c) { return r * LDT + c; }

// LOGITS: the gate arrives as bf16 logits (fused gate activation) instead of fp32 g.
template <typename TOut, bool LOGITS>
__global__ void __launch_bounds__(NT + 32, 1)
    prefill_tc_kernel(const PrefillParams p, const __grid_constant__ TcMaps maps) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char *sm = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float *sEgr = reinterpret_cast<float *>(sm + OFF_EGR);
  float *sSeg = reinterpret_cast<float *>(sm + OFF_SEG);
  float *sGr2 = reinterpret_cast<float *>(sm + OFF_GR2);
  float *sB = reinterpret_cast<float *>(sm + OFF_BETA);
  uint64_t *bars = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
  uint64_t *bar_tma = bars + 0;      // TMA -> workers: raw tiles landed
  uint64_t *bar_raw = bars + 1;      // workers -> control: raw tiles consumed (16 warps)
  uint64_t *bar_opsap = bars + 2;    // workers -> control: A|P operands built (16 warps)
  uint64_t *bar_y = bars + 3;        // control -> workers: Y^T product done (S^T read)
  uint64_t *bar_ops = bars + 4;      // workers -> control: T Diag(beta) ready, S^T scaled
  uint64_t *bar_ap = bars + 5;       // control -> workers: O^T and A|P products done
  uint64_t *bar_u = bars + 6;        // control -> control: U^T product done
  uint64_t *bar_mma = bars + 7;      // control -> workers: chunk's last products done
  uint64_t *bar_st = bars + 8;       // workers -> control: chunk staged, previous O^T stored
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(bars + 9);
  volatile int *s_abort = reinterpret_cast<volatile int *>(s_tmem + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane_id = tid & 31;
  const bool control = warp == NT / 32;            // warp 16: TMA and MMA issue
  const int l = ((warp & 3) << 5) | lane_id;       // TMEM lane of a worker thread
  const int g = (warp >> 2) & 3;                   // worker column quarter
  const uint32_t lane = (uint32_t)((warp & 3) * 32) << 16;
  const int H = p.H;
  // Local-state mode (context-parallel pass 1): CTA part 0 runs the segment from a
  // zero state with its values (-> S_loc), part 1 from the identity with zero values
  // (-> M = A_L ... A_1); the two are the column blocks of the augmented state.
  const int pairs = p.n_req * H;
  const int part = p.local_mode ? (int)(blockIdx.x / pairs) : 0;
  const int rem = (int)(blockIdx.x % pairs);
  const int r = p.order ? p.order[rem / H] : rem / H;
  const int h = rem % H;
  const bool load_q = !p.local_mode;
  constexpr bool logits = LOGITS;
  const bool zero_v = p.local_mode && part == 1;
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
    mbar_init(bar_raw, NT / 32);
    mbar_init(bar_opsap, NT / 32);
    mbar_init(bar_ops, NT / 32);
    mbar_init(bar_ap, 1);
    mbar_init(bar_y, 1);
    mbar_init(bar_u, 1);
    mbar_init(bar_mma, 1);
    mbar_init(bar_st, NT / 32);
    *s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = *s_tmem;
  const int n_chunks = (len + C - 1) / C;

  if (control) {
    // ======================= control warp: TMA + MMA issue =======================
    if (lane_id == 0) {
      tma_prefetch_desc(&maps.q);
      tma_prefetch_desc(&maps.k);
      tma_prefetch_desc(&maps.v);
      tma_prefetch_desc(&maps.g);
      auto issue_tma = [&](int c0) {
        mbar_expect_tx(bar_tma, RAW_BYTES - (load_q ? 0u : 16384u) - (logits ? 16384u : 0u));
        const int y = bos + c0;
        for (int half = 0; half < 2; ++half) {
          const int x = h * DH + 64 * half;
          tma_load_2d(sm + OFF_KRAW + 8192 * half, &maps.k, x, y, bar_tma);
          if (load_q) tma_load_2d(sm + OFF_QRAW + 8192 * half, &maps.q, x, y, bar_tma);
          tma_load_2d(sm + OFF_VRAW + 8192 * half, &maps.v, x, y, bar_tma);
        }
        if (logits) {
          for (int half = 0; half < 2; ++half)
            tma_load_2d(sm + OFF_GRAW + 8192 * half, &maps.g, h * DH + 64 * half, y, bar_tma);
        } else {
          for (int qd = 0; qd < 4; ++qd)
            tma_load_2d(sm + OFF_GRAW + 8192 * qd, &maps.g, h * DH + 32 * qd, y, bar_tma);
        }
      };
      uint32_t ph_raw = 0, ph_opsap[1] = {0}, ph_ops = 0, ph_u = 0, ph_st = 0;
      auto cwait = [&](uint64_t *bar, uint32_t &ph) -> bool {
        const bool good = *s_abort == 0 && mbar_wait(bar, ph);
        ph ^= 1u;
        if (!good) {
          *s_abort = 1;
          set_status(p.status, STATUS_TIMEOUT);
        }
        tc_fence_after();
        return good;
      };
      if (n_chunks > 0) issue_tma(0);
      for (int ci = 0; ci < n_chunks; ++ci) {
        // O^T = S^T (gamma Q)^T needs only the state and gamma*Q: issue it as soon as the
        // chunk is staged, so it runs while the workers build the A|P operands
        if (!cwait(bar_st, ph_st)) break;
        {
          const uint32_t id = idesc_tf32(64);
          const uint32_t qb = smem_u32(sm + OFF_GQ);
#pragma unroll
          for (int s = 0; s < DH / 8; ++s)
            mma_tf32_ts(tm + TM_O, tm + TM_S + 8 * s, sw128_desc(qb, C, s), id, s > 0);
        }
        // A | P: row block b against its R'_b (N = 32(b+1)), each over the two halves of
        // the key channels into its own accumulator: four interleaved chains of 8 steps
        if (!cwait(bar_opsap, ph_opsap[0])) break;
        {
          const uint32_t rp = smem_u32(sm);
#pragma unroll
          for (int s = 0; s < DH / 16; ++s) {
#pragma unroll
            for (int half = 0; half < 2; ++half)
#pragma unroll
              for (int b = 0; b < 2; ++b) {
                const int ks = (DH / 16) * half + s;
                mma_tf32_ts(tm + ap_col(b, half), tm + TM_L + 8 * ks,
                            sw128_desc(rp + rp_off(b), 32 * (b + 1), ks), idesc_tf32(32 * (b + 1)),
                            s > 0);
              }
          }
          mma_commit(bar_ap);  // gamma*Q and the R'_b operands are free after this
        }
        // raw tiles consumed, V^T in TMEM, gamma*K in shared memory
        if (!cwait(bar_raw, ph_raw)) break;
        if (ci + 1 < n_chunks) issue_tma((ci + 1) * C);
        {  // Y^T = V^T - S^T (gamma K)^T, while the workers solve T
          const uint32_t idn = idesc_tf32(64, true);
          const uint32_t kb = smem_u32(sm + OFF_GQ);
#pragma unroll
          for (int s = 0; s < DH / 8; ++s)
            mma_tf32_ts(tm + TM_L, tm + TM_S + 8 * s, sw128_desc(kb, C, s), idn, true);
          mma_commit(bar_y);
        }
        if (!cwait(bar_ops, ph_ops)) break;  // T Diag(beta) ready, S^T scaled by gamma_63
        {  // U^T = Y^T (T Diag(beta))^T
          const uint32_t id = idesc_tf32(64);
          const uint32_t tb = smem_u32(sm + OFF_TB);
#pragma unroll
          for (int s = 0; s < C / 8; ++s)
            mma_tf32_ts(tm + TM_X2, tm + TM_L + 8 * s, sw128_desc(tb, C, s), id, s > 0);
          mma_commit(bar_u);
        }
        // U^T is the A operand of the last two products: wait for it to land
        if (!cwait(bar_u, ph_u)) break;
        {
          const uint32_t id64 = idesc_tf32(64), id128 = idesc_tf32(128);
          const uint32_t pb = smem_u32(sm + OFF_P), kb = smem_u32(sm + OFF_KHT);
#pragma unroll
          for (int s = 0; s < C / 8; ++s) {
            mma_tf32_ts(tm + TM_O, tm + TM_X2 + 8 * s, sw128_desc(pb, C, s), id64, true);
            mma_tf32_ts(tm + TM_S, tm + TM_X2 + 8 * s, sw128_desc(kb, DH, s), id128, true);
          }
          mma_commit(bar_mma);
        }
      }
    }
  } else {
    // ======================= 16 worker warps =======================
    uint32_t ph_tma = 0, ph_ap[1] = {0}, ph_y = 0, ph_mma = 0;
    auto wsync = [&]() { named_sync(1, NT); };
    // every worker waits, then the workers synchronise so an abort is seen by all
    auto wwait = [&](uint64_t *bar, uint32_t &ph) -> bool {
      if (!(*s_abort == 0 && mbar_wait(bar, ph))) {
        *s_abort = 1;
        set_status(p.status, STATUS_TIMEOUT);
      }
      ph ^= 1u;
      wsync();
      tc_fence_after();
      return *s_abort == 0;
    };
    // one arrival per warp once all its lanes' writes are visible to the async proxy
    auto warp_arrive = [&](uint64_t *bar) {
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane_id == 0) mbar_arrive(bar);
    };

    // initial state -> S^T in TMEM (lane v holds S[:, v])
    {
      const float *s0 =
          p.initial_state ? p.initial_state + ((size_t)(r * H + h)) * DH * DH : nullptr;
      float v[32];
#pragma unroll
      for (int j = 0; j < 32; ++j)
        v[j] = p.local_mode ? ((part == 1 && 32 * g + j == l) ? 1.f : 0.f)
                            : (s0 ? s0[(size_t)(32 * g + j) * DH + l] : 0.f);
      tmem_st32(tm + lane + TM_S + 32 * g, v);
      tmem_wait_st();
    }

    // beta of the chunk about to start, loaded one chunk ahead (threads 0..63)
    auto load_beta = [&](int c0) -> float {
      float b = 0.f;
      if (tid < C && c0 + tid < len) {
        b = p.beta[(size_t)(bos + c0 + tid) * H + h];
        if (p.validate && !(b >= 0.f && b <= 1.f)) set_status(p.status, STATUS_GATE_RANGE);
      }
      return b;
    };
    float beta_next = load_beta(0);
    // T Diag(beta) is lower triangular: its blocks above the diagonal stay zero, so they
    // are written once here; the solve below stores every other element as it finalises it
    for (int e = tid; e < C * C / 4; e += NT)
      reinterpret_cast<float4 *>(sm + OFF_TB)[e] = make_float4(0.f, 0.f, 0.f, 0.f);
    // Stage a chunk: its beta, wait for its tiles, cumulative gate, row operands
    // (L* into TMEM, R into scratch, gamma*Q).  Chunk n+1 is staged while chunk n's
    // last MMAs run.
    auto stage = [&](int cs) -> bool {
      const int c0 = cs * C;
      const int n = min(C, len - c0);
      if (tid < C) sB[tid] = beta_next;
      if (!wwait(bar_tma, ph_tma)) return false;
      beta_next = load_beta(c0 + C);

      // ---- a2: cumulative gate (thread = channel l, tokens 16g..16g+15) --------
      // Every thread reads its raw gates before the first worker sync and writes the
      // cumulative ones only after it, so the bf16 logits can share the region.
      {
        float gv[16];
        if (logits) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int t = 16 * g + j;
            gv[j] = (t < n) ? gate_from_logit(bf16_at(sm + OFF_GRAW, t, l)) : 0.f;
          }
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int t = 16 * g + j;
            gv[j] = (t < n) ? *reinterpret_cast<const float *>(sm + OFF_GRAW + g_off(t, l)) : 0.f;
          }
        }
        if (p.validate && !logits)
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (!(gv[j] >= kGateLower && gv[j] <= 0.f)) set_status(p.status, STATUS_GATE_RANGE);
#pragma unroll
        for (int j = 1; j < 16; ++j) gv[j] += gv[j - 1];
        sSeg[g * DH + l] = gv[15];
        wsync();
        float off = 0.f;
        for (int gg = 0; gg < g; ++gg) off += sSeg[gg * DH + l];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          gv[j] = (gv[j] + off) * LOG2E;
          *reinterpret_cast<float *>(sm + OFF_GRAW + g_off(16 * g + j, l)) = gv[j];
        }
        sGr2[g * DH + l] = gv[15];
        sEgr[g * DH + l] = ex2(gv[15]);
        wsync();
      }

      // ---- a3 operands (thread = row i, channels 32g..32g+31) -----------------
      // L*_i = x_i exp(G_i - G_m) with m = 32 b + 15 the reference row of i's 32-row block
      // (x = k or q) goes to TMEM; K side: k_i to fp32 scratch (for R'_b); Q side:
      // gamma*Q = L* exp(G_m) to its B operand.
      const bool kside = l < C;
      const int i = l & (C - 1);
      const int bi = 2 * (i >> 5);  // the 16-row group ending at the reference row of i's block
      const bool valid = i < n && (kside || load_q);
      float *Rs = reinterpret_cast<float *>(sm + OFF_R);  // [64][LDR] fp32 scratch
      {
        const unsigned char *xraw = sm + (kside ? OFF_KRAW : OFF_QRAW);
        const int rb = 16 * bi + 15;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          float Lv[16];
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            const int c = 32 * g + 16 * half + 4 * c4;
            const float4 gi = *reinterpret_cast<const float4 *>(sm + OFF_GRAW + g_off(i, c));
            const float4 grb = *reinterpret_cast<const float4 *>(sm + OFF_GRAW + g_off(rb, c));
            float x[4];
            bf16_x4(xraw, i, c, x);
            const float giv[4] = {gi.x, gi.y, gi.z, gi.w}, grv[4] = {grb.x, grb.y, grb.z, grb.w};
            float lst[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              if (!valid) x[e] = 0.f;
              lst[e] = x[e] * ex2(giv[e] - grv[e]);
              Lv[4 * c4 + e] = tf32_rna(lst[e]);
            }
            if (kside) {  // k itself: R'_b takes its block factor in one exponential
              *reinterpret_cast<float4 *>(&Rs[i * LDR + c]) = make_float4(x[0], x[1], x[2], x[3]);
            } else {
              const float4 eg = *reinterpret_cast<const float4 *>(&sEgr[bi * DH + c]);
              *reinterpret_cast<float4 *>(sm + OFF_GQ + sw128_chunk(C, i, c)) =
                  make_float4(tf32_rna(lst[0] * eg.x), tf32_rna(lst[1] * eg.y),
                              tf32_rna(lst[2] * eg.z), tf32_rna(lst[3] * eg.w));
            }
          }
          tmem_st16(tm + lane + TM_L + 32 * g + 16 * half, Lv);
        }
      }
      return true;
    };
    bool ok = n_chunks > 0 ? stage(0) : true;
    for (int ci = 0; ci < n_chunks && ok; ++ci) {
      const int c0 = ci * C;
      const int n = min(C, len - c0);
      const bool kside = l < C;
      const int i = l & (C - 1);
      float *Rs = reinterpret_cast<float *>(sm + OFF_R);  // [64][LDR] fp32 scratch
      warp_arrive(bar_st);  // gamma*Q built, the previous chunk's O^T read: -> O^T
      // thread = channel l, tokens 16g..16g+15: V^T and gamma*K (kept in registers until
      // L* and gamma*Q are free), Khat^T = k exp(G_63 - G) straight to its B operand
      uint32_t vT2[8];
      float gkT[16];
      {
        const float G63 = *reinterpret_cast<const float *>(sm + OFF_GRAW + g_off(C - 1, l));
        float kh[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int t = 16 * g + j;
          const float G2 = *reinterpret_cast<const float *>(sm + OFF_GRAW + g_off(t, l));
          const uint32_t vb = (t < n && !zero_v) ? (uint32_t)*reinterpret_cast<const unsigned short *>(
                                            sm + OFF_VRAW + bf16_off(t, l))
                                      : 0u;
          if (j & 1) vT2[j >> 1] |= vb << 16; else vT2[j >> 1] = vb;
          const float kk = (t < n) ? bf16_at(sm + OFF_KRAW, t, l) : 0.f;
          gkT[j] = tf32_rna(kk * ex2(G2));
          kh[j] = tf32_rna(kk * ex2(G63 - G2));
        }
#pragma unroll
        for (int m4 = 0; m4 < 4; ++m4)
          *reinterpret_cast<float4 *>(sm + OFF_KHT + sw128_chunk(DH, l, 16 * g + 4 * m4)) =
              make_float4(kh[4 * m4], kh[4 * m4 + 1], kh[4 * m4 + 2], kh[4 * m4 + 3]);
      }
      wsync();  // every raw tile read: the raw region now takes the R'_b operands
      // R'_b row j = k_j exp(G_mb - G_j) for the rows j of blocks up to b, m_b = 32 b + 15
      // (the 16-row group end 2b of the G table), spread over all workers.  One exponential
      // of the exponent difference: a factor underflows only where the true factor is
      // below FLT_MIN, and then its product with an L* factor (<= exp(75)) is < exp(-12).
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        const int rows = 32 * (b + 1);
        for (int it = tid; it < rows * 32; it += NT) {
          const int j = it >> 5, c = (it & 31) * 4;
          const float4 kv = *reinterpret_cast<const float4 *>(&Rs[j * LDR + c]);
          const float4 gj = *reinterpret_cast<const float4 *>(sm + OFF_GRAW + g_off(j, c));
          const float4 gm = *reinterpret_cast<const float4 *>(&sGr2[(2 * b) * DH + c]);
          *reinterpret_cast<float4 *>(sm + rp_off(b) + sw128_chunk(rows, j, c)) =
              make_float4(tf32_rna(kv.x * ex2(gm.x - gj.x)), tf32_rna(kv.y * ex2(gm.y - gj.y)),
                          tf32_rna(kv.z * ex2(gm.z - gj.z)), tf32_rna(kv.w * ex2(gm.w - gj.w)));
        }
      }
      tmem_wait_st();
      warp_arrive(bar_opsap);  // -> A|P MMAs
      if (!(ok = wwait(bar_ap, ph_ap[0]))) break;
      {
        float vT[16];
#pragma unroll
        for (int j = 0; j < 16; ++j)
          vT[j] = __uint_as_float((j & 1) ? (vT2[j >> 1] & 0xFFFF0000u) : (vT2[j >> 1] << 16));
        tmem_st16(tm + lane + TM_L + 16 * g, vT);  // L* is dead: V^T starts Y^T
      }
      // gamma*Q has been read by the O^T product: its tile takes gamma*K (rows = tokens)
#pragma unroll
      for (int j = 0; j < 16; ++j)
        *reinterpret_cast<float *>(sm + OFF_GQ + sw128_offset(C, 16 * g + j, l)) = gkT[j];
      tmem_wait_st();
      warp_arrive(bar_raw);  // R'_b consumed (next TMA may start); V^T and gamma*K ready

      // ---- a4: T = (I + Diag(beta) A)^-1 (blocked, fp32), P operand ------------
      float *Ms = reinterpret_cast<float *>(sm + OFF_MS);
      float *Ti = reinterpret_cast<float *>(sm + OFF_TI);
      float *Ys = reinterpret_cast<float *>(sm + OFF_Y);
      // element (r, c) of T Diag(beta), the B operand of U^T, once T_rc is final
      auto put_tb = [&](int r, int c, float t) {
        *reinterpret_cast<float *>(sm + OFF_TB + sw128_offset(C, r, c)) = tf32_rna(t * sB[c]);
      };
      {
        // this warp's 32 rows are one row block: the sum of its two accumulators (columns
        // past the block's width belong to other accumulators and are masked below)
        const int blk = warp & 1;
        float a[16], a_hi[16];
        tmem_ld16(tm + lane + ap_col(blk, 0) + 16 * g, a);
        tmem_ld16(tm + lane + ap_col(blk, 1) + 16 * g, a_hi);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j) a[j] += a_hi[j];
        if (kside) {
          const float bi_ = sB[i];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int c = 16 * g + j;
            Ms[rot(i, c)] = (c < i) ? bi_ * a[j] : 0.f;
          }
        } else {
#pragma unroll
          for (int j = 0; j < 16; j += 4) {
            const int c = 16 * g + j;
            *reinterpret_cast<float4 *>(sm + OFF_P + sw128_chunk(C, i, c)) =
                make_float4(c + 0 <= i ? tf32_rna(a[j]) : 0.f, c + 1 <= i ? tf32_rna(a[j + 1]) : 0.f,
                            c + 2 <= i ? tf32_rna(a[j + 2]) : 0.f,
                            c + 3 <= i ? tf32_rna(a[j + 3]) : 0.f);
          }
        }
      }
      wsync();
      // diagonal 32x32 blocks: forward substitution, x_k = [k == j] - sum_{q<k} N_kq x_q for
      // column j.  Warp w takes block w / 8 and its columns w % 8 + 8 c (c < 4) as four
      // chains over the same rows, so the one value N_kq of a step (lane k) feeds all four
      // and the chains' shuffles overlap; the next step's N_kq is loaded a step ahead.
      {
        const int o = 32 * (warp >> 3), k = lane_id;
        int jj[4];
        float x[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          jj[c] = (warp & 7) + 8 * c;
          x[c] = (k == jj[c]) ? 1.f : 0.f;
        }
        float m_next = Ms[rot(o + k, o)];
#pragma unroll
        for (int q = 0; q < 31; ++q) {
          const float m = m_next;
          if (q < 30) m_next = Ms[rot(o + k, o + q + 1)];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const float xq = __shfl_sync(0xffffffffu, x[c], q);
            if (q >= jj[c] && k > q) x[c] -= m * xq;
          }
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float t = (k >= jj[c]) ? x[c] : 0.f;
          Ti[rot(o + k, o + jj[c])] = t;
          put_tb(o + k, o + jj[c], t);
        }
      }
      wsync();
      // 32 -> 64: T[32:64, 0:32] = -T[32:64, 32:64] (N[32:64, 0:32] T[0:32, 0:32]);
      // two outputs per thread, each summed in two halves to shorten the FMA chains
      {
        const int ii = tid >> 4, j0 = tid & 15;  // rows ii, columns j0 and j0 + 16
        float y0a = 0.f, y0b = 0.f, y1a = 0.f, y1b = 0.f;
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const float na = Ms[rot(32 + ii, q)], nb = Ms[rot(32 + ii, q + 16)];
          if (q >= j0) y0a += na * Ti[rot(q, j0)];
          y0b += nb * Ti[rot(q + 16, j0)];
          y1b += (q >= j0) ? nb * Ti[rot(q + 16, j0 + 16)] : 0.f;
          (void)y1a;
        }
        Ys[ii * 33 + j0] = y0a + y0b;
        Ys[ii * 33 + j0 + 16] = y1b;
        wsync();
        float t0a = 0.f, t0b = 0.f, t1a = 0.f, t1b = 0.f;
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          if (q <= ii) {
            const float tv = Ti[rot(32 + ii, 32 + q)];
            t0a += tv * Ys[q * 33 + j0];
            t1a += tv * Ys[q * 33 + j0 + 16];
          }
          if (q + 16 <= ii) {
            const float tv = Ti[rot(32 + ii, 48 + q)];
            t0b += tv * Ys[(q + 16) * 33 + j0];
            t1b += tv * Ys[(q + 16) * 33 + j0 + 16];
          }
        }
        put_tb(32 + ii, j0, -(t0a + t0b));
        put_tb(32 + ii, j0 + 16, -(t1a + t1b));
      }
      // ---- S^T <- S^T Diag(gamma_63) once the O^T and Y^T products have read S^T ----
      if (!(ok = wwait(bar_y, ph_y))) break;
      {
        float v[32];
        tmem_ld32(tm + lane + TM_S + 32 * g, v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] *= sEgr[3 * DH + 32 * g + j];
        tmem_st32(tm + lane + TM_S + 32 * g, v);
        tmem_wait_st();
      }
      warp_arrive(bar_ops);  // -> U^T, then O^T += U^T P^T, S^T += U^T Khat
      if (ci + 1 < n_chunks && !(ok = stage(ci + 1))) break;  // overlaps those MMAs
      if (!(ok = wwait(bar_mma, ph_mma))) break;

      // ---- a6: outputs (lane = value channel, tokens 16g..) and snapshots -------
      if (go) {
        float o[16];
        tmem_ld16(tm + lane + TM_O + 16 * g, o);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int t = 16 * g + j;
          if (t < n) store_elem(go, ((size_t)(bos + c0 + t) * H + h) * DH + l, o[j]);
        }
      }
      if (snaps_ok && n == C && (c0 + C) % p.snapshot_stride == 0) {
        const size_t row = (size_t)p.cu_snapshots[r] + (c0 + C) / p.snapshot_stride - 1;
        float *dst = p.snapshots + (row * H + h) * (size_t)DH * DH;
        float v[32];
        tmem_ld32(tm + lane + TM_S + 32 * g, v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) dst[(size_t)(32 * g + j) * DH + l] = v[j];
      }
      tc_fence_before();
      wsync();
    }

    float *fin = p.local_mode ? (part == 0 ? p.s_loc : p.m) : p.final_state;
    if (ok && fin) {
      float *dst = fin + ((size_t)(r * H + h)) * DH * DH;
      tc_fence_after();
      float v[32];
      tmem_ld32(tm + lane + TM_S + 32 * g, v);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 32; ++j) dst[(size_t)(32 * g + j) * DH + l] = v[j];
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*s_abort && tid == 0) {
    // the CTA gave up: give in-flight copies and MMAs a bounded chance to land
    mbar_wait(bar_tma, 0, 100000000ull);
    mbar_wait(bar_tma, 1, 100000000ull);
    mbar_wait(bar_y, 0, 100000000ull);
    mbar_wait(bar_y, 1, 100000000ull);
    mbar_wait(bar_u, 0, 100000000ull);
    mbar_wait(bar_u, 1, 100000000ull);
    mbar_wait(bar_mma, 0, 100000000ull);
    mbar_wait(bar_mma, 1, 100000000ull);
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_relinquish();
    tmem_dealloc(tm, TM_COLS);
  }
}

// The driver's tensor-map encoder, looked up through the runtime so that the
// library does not link libcuda (it loads on machines without a driver).
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

bool encode_map(CUtensorMap *m, const void *ptr, CUtensorMapDataType dt, uint64_t esize,
                uint64_t inner, uint64_t rows, uint32_t box_inner) {
  const EncodeTiledFn encode = encode_tiled_fn();
  if (!encode) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * esize};
  cuuint32_t box[2] = {box_inner, 64};
  cuuint32_t es[2] = {1, 1};
  return encode(m, dt, 2, const_cast<void *>(ptr), dims, strides, box, es,
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
  if (!encode_map(&maps.q, p.q ? p.q : p.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, W, T, 64) ||
      !encode_map(&maps.k, p.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, W, T, 64) ||
      !encode_map(&maps.v, p.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, W, T, 64) ||
      !(p.g_logits ? encode_map(&maps.g, p.g_logits, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, W, T, 64)
                   : encode_map(&maps.g, p.g, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, W, T, 32)))
    return cudaErrorInvalidValue;
  const unsigned grid = (unsigned)(p.n_req * p.H * (p.local_mode ? 2 : 1));
  auto run = [&](auto kernel) -> cudaError_t {
    const cudaError_t e =
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    kernel<<<grid, NT + 32, SMEM_ALLOC, stream>>>(p, maps);
    return cudaGetLastError();
  };
  const bool logits = p.g_logits != nullptr;
  if (out_dtype == KDA_BF16)
    return logits ? run(prefill_tc_kernel<__nv_bfloat16, true>)
                  : run(prefill_tc_kernel<__nv_bfloat16, false>);
  return logits ? run(prefill_tc_kernel<float, true>) : run(prefill_tc_kernel<float, false>);
}

}  // namespace kda

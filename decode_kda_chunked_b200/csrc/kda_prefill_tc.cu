// Chunked KDA prefill on the sm_100a tensor cores: TMA tile loads, tcgen05
// tf32 MMAs with fp32 accumulators in tensor memory (TMEM), fp32 SIMT for the
// cumulative gate, the exponentials and the triangular solve.
//
// The chunk algebra is that of the chunk-parallel form (tokens of a chunk in
// parallel, state passed between chunks in order: "Kimi K3 开源日来了",
// FlashKDA section), here with chunks of 32 tokens, written transposed so that
// every MMA has M = 128 with one TMEM lane per feature channel (S^T, U^T, O^T
// have lanes = value channels, columns = key channels or tokens):
//
//   A | P   [128 x 32] = [L_k ; L_q] R'^T                 (A from TMEM, lanes 0-31 | 32-63)
//   O^T     = S^T (gamma*Q)^T                            (A = S^T in TMEM)
//   Y^T     = V^T - S^T (gamma*K)^T                      (A = S^T in TMEM, D starts as V^T)
//   U^T     = Y^T (T Diag(b))^T                          (A = Y^T in TMEM)
//   O^T    += U^T P^T,   S^T <- S^T Diag(gamma_31) + U^T Khat      (A = U^T in TMEM)
// U = T Diag(b) (V - (gamma*K) S) is the chunk form's U~ - W S with W never formed.
//
// Gate factorisation for A and P: exp(G_i - G_j) = exp(G_i - G_15) exp(G_15 - G_j) with
// the chunk's row 15 as reference.  The left factor is <= exp(5 * 15) (rows i < 15) or
// <= 1, the right factor <= exp(5 * 16) (columns j > 15) or <= 1.  Because
// log alpha >= -5 (the lower-bounded decay of KDA, CSDN post on the Kimi K3 technical
// report, section 一.1) every factor is a finite fp32 number; only masked products
// (j > i) can overflow, and they are dropped by selection, never multiplied.
// gamma_i = exp(G_i) is exp(G_i - G_15) exp(G_15), a product of two finite factors
// that is flushed to zero only where the true value is below FLT_MIN.
//
// All tensor-core operands are tf32 (B operands K-major with the 128-byte swizzle in
// shared memory, rounded to nearest even): bf16 operands for the gate-scaled products
// would cost about 2e-3 of relative accuracy, tf32 stays near 5e-4.
//
// Warp roles.  One CTA runs one (request, head) chain: two control warps issue every
// TMA load and tcgen05.mma, and two groups of 8 worker warps run side by side,
// handing off through mbarriers (intra-chunk work in parallel with the state
// passing, as the FlashKDA section of "Kimi K3 开源日来了" describes):
//
//   group A (warps 0-7), chunk m:  gate(m): cumulative gate;  rows(m): L_k, L_q -> TMEM,
//       R', gamma*Q, gamma*K -> smem  [-> A|P(m)];  read(m): Diag(b) A, P;
//       solve(m): T Diag(b)  [-> U^T(m)]
//   group B (warps 8-15), chunk n:  scale(n): S^T *= gamma_31 once O^T, Y^T(n) read S^T
//       [-> last products(n)];  khat(n+1): Khat^T;  out(n): O^T -> o, snapshot;
//       vt(n+1): V^T -> TMEM  [with group A's read(n+1): -> O^T, Y^T(n+1)]
//
// so group A prepares chunk n+1 while group B finishes chunk n, and every product
// runs while the workers do other work.  Khat^T, P and T Diag(b) are double
// buffered by chunk parity, raw tiles too (chunk m+2 loads as soon as chunk m's
// tiles are read); every other buffer is rewritten only after the product that
// reads it has completed (group A starts chunk m after O^T, Y^T(m-1)).  Every wait
// is bounded; a wait that runs out ends the CTA with KDA_ERR_TIMEOUT in the status
// word, after the CTA has let every copy and product it issued land.
#include "kda_internal.cuh"
#include "kda_sm100.cuh"

namespace kda {
namespace {

using namespace sm100;

// The bounded wait with its slow path (suspend, clock and abort checks) out of line:
// one copy in the kernel's code instead of one per wait site, since the kernel's
// speed depends on how much of its code the instruction caches hold.
__device__ __noinline__ bool mbar_wait_slow(uint64_t *bar, uint32_t parity, uint64_t timeout_ns,
                                            const volatile int *abort_flag) {
  return mbar_wait(bar, parity, timeout_ns, abort_flag);
}
__device__ __forceinline__ bool mbar_wait_ni(uint64_t *bar, uint32_t parity, uint64_t timeout_ns,
                                             const volatile int *abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  return mbar_wait_slow(bar, parity, timeout_ns, abort_flag);
}


constexpr int C = 32;     // tokens per chunk of this kernel
constexpr int DH = 128;   // head dim (dk = dv)
constexpr int NT = 512;   // worker threads per CTA: 16 warps (plus one control warp)
constexpr int NA = 256;   // group A threads (warps 0-7); group B is warps 8-15
constexpr int MREF = 15;  // reference row of the gate factorisation
constexpr float LOG2E = 1.4426950408889634f;

// ---- shared memory map (byte offsets from a 1024-aligned base) ----
// Raw tiles of one chunk: q, k, v bf16 [32 x 128] as two 64-column 128B-swizzled TMA
// boxes each; g fp32 [32 x 128] as four 32-column boxes (bf16 gate logits: two
// 64-column boxes).  Chunk m uses buffer m & 1.
constexpr uint32_t RAW_BYTES = 40960;
constexpr uint32_t R_K = 0, R_Q = 8192, R_V = 16384, R_G = 24576;
constexpr uint32_t OFF_RAW = 0;
constexpr uint32_t OFF_GQ = 81920;   // gamma*Q  tf32 B operand [32 x 128]
constexpr uint32_t OFF_GK = 98304;   // gamma*K  tf32 B operand [32 x 128]
constexpr uint32_t OFF_KH = 114688;  // Khat^T   tf32 B operand [128 x 32], x2 (chunk parity)
constexpr uint32_t OFF_RP = 147456;  // R'       tf32 B operand [32 x 128]
constexpr uint32_t OFF_PP = 163840;  // P        tf32 B operand [32 x 32], x2
constexpr uint32_t OFF_TB = 172032;  // T Diag(beta) tf32 B operand [32 x 32], x2
constexpr uint32_t OFF_NS = 180224;  // Diag(beta) A, strict lower, fp32 [32][LDN]
constexpr int LDN = 36;
constexpr uint32_t OFF_TS = 184832;  // the two diagonal 16x16 blocks of T, fp32 [32][LDN]
constexpr uint32_t OFF_XS = 189440;  // N10 T00, fp32 [16][LDX]
constexpr int LDX = 20;
constexpr uint32_t OFF_GC = 190720;  // exp(G_31) per key channel, [4][128] (chunk index mod 4)
constexpr uint32_t OFF_BT = 192768;  // beta [2][32] (chunk parity)
constexpr uint32_t OFF_SEG = 193024; // spare [2][128]
constexpr uint32_t OFF_BAR = 194048; // mbarriers, TMEM base, flags (+ phase counters)
// Cumulative gate log2(e) G of a chunk, fp32 [32 tokens][LDG], x2 (chunk parity): rows
// padded to LDG = 132 floats, so that eight consecutive channels of a token are one
// 16-byte aligned pair of loads at a plain offset, and lanes reading eight rows hit
// eight distinct bank quads.
constexpr uint32_t OFF_GT = 194304;
constexpr int LDG = 132;
constexpr uint32_t GT_BYTES = C * LDG * 4;
constexpr uint32_t SMEM_BYTES = OFF_GT + 2 * GT_BYTES;
constexpr uint32_t SMEM_ALLOC = SMEM_BYTES + 1024;  // alignment slack
static_assert(OFF_RAW + 2 * RAW_BYTES == OFF_GQ, "raw buffers");
static_assert(OFF_GQ % 1024 == 0 && OFF_GK % 1024 == 0 && OFF_KH % 1024 == 0 &&
                  OFF_RP % 1024 == 0 && OFF_PP % 1024 == 0 && OFF_TB % 1024 == 0,
              "swizzled operands need 1024-byte alignment");
static_assert(OFF_GQ + 16384 == OFF_GK && OFF_GK + 16384 == OFF_KH &&
                  OFF_KH + 2 * 16384 == OFF_RP && OFF_RP + 16384 == OFF_PP &&
                  OFF_PP + 2 * 4096 == OFF_TB && OFF_TB + 2 * 4096 == OFF_NS,
              "operand tiles");
static_assert(OFF_NS + C * LDN * 4 == OFF_TS && OFF_TS + C * LDN * 4 == OFF_XS &&
                  OFF_XS + 16 * LDX * 4 == OFF_GC && OFF_GC + 4 * DH * 4 == OFF_BT &&
                  OFF_BT + 2 * C * 4 == OFF_SEG &&
                  OFF_SEG + 2 * DH * 4 == OFF_BAR && OFF_BAR + 256 == OFF_GT,
              "scratch tiles");
static_assert(SMEM_BYTES + 1024 <= 232448, "227 KB of shared memory per CTA");
__host__ __device__ constexpr uint32_t kh_off(int m) { return OFF_KH + 16384u * (m & 1); }
__host__ __device__ constexpr uint32_t pp_off(int m) { return OFF_PP + 4096u * (m & 1); }
__host__ __device__ constexpr uint32_t tb_off(int m) { return OFF_TB + 4096u * (m & 1); }

// ---- TMEM column map (512 columns x 128 lanes of fp32) ----
constexpr uint32_t TM_S = 0;     // S^T (lane = value channel, col = key channel)
constexpr uint32_t TM_L = 128;   // [L_k ; L_q]: A operand of A|P (lanes 0-31 | 32-63)
constexpr uint32_t TM_AP = 256;  // A (lanes 0-31) | P (lanes 32-63), 32 columns
constexpr uint32_t TM_Y = 288;   // V^T -> Y^T
constexpr uint32_t TM_U = 320;   // U^T
constexpr uint32_t TM_O = 352;   // O^T (local state: Y_M^T)
constexpr uint32_t TM_M = 384;   // local state: M^T, the segment's transition
constexpr uint32_t TM_COLS = 512;

struct TcMaps {
  CUtensorMap q, k, v, g;
};

// bf16 [32 x 128] tile: byte offset of the 16-byte chunk with channels c..c+7 (c % 8 == 0)
// of row t, and of one element
__device__ __forceinline__ uint32_t bf16_chunk(int t, int c) {
  return (uint32_t)(c >> 6) * 4096u + (uint32_t)t * 128u +
         ((uint32_t)(((c & 63) >> 3) ^ (t & 7)) << 4);
}
__device__ __forceinline__ uint32_t bf16_off(int t, int c) {
  return bf16_chunk(t, c & ~7) + (uint32_t)(c & 7) * 2u;
}
__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }
__device__ __forceinline__ void bf16_x8(const uint4 u, float *x) {
  x[0] = bf16_lo(u.x); x[1] = bf16_hi(u.x); x[2] = bf16_lo(u.y); x[3] = bf16_hi(u.y);
  x[4] = bf16_lo(u.z); x[5] = bf16_hi(u.z); x[6] = bf16_lo(u.w); x[7] = bf16_hi(u.w);
}
__device__ __forceinline__ float bf16_at(const unsigned char *tile, int t, int c) {
  return bf16_lo(*reinterpret_cast<const unsigned short *>(tile + bf16_off(t, c)));
}
// fp32 [32 x 128] tile as four 32-column boxes
__device__ __forceinline__ uint32_t f32_off(int t, int c) {
  return (uint32_t)(c >> 5) * 4096u + (uint32_t)t * 128u +
         ((uint32_t)(((c & 31) >> 2) ^ (t & 7)) << 4) + (uint32_t)(c & 3) * 4u;
}
// eight consecutive channels c..c+7 (c % 8 == 0) of token t of a gate table (row stride LDG)
__device__ __forceinline__ void ld8g(const float *table, int t, int c, float *x) {
  const float4 *q = reinterpret_cast<const float4 *>(table + t * LDG + c);
  const float4 a = q[0], b = q[1];
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}
// fp32 -> tf32, round to nearest even (the tensor cores read the 19 leading bits)
__device__ __forceinline__ float tf32_rn(float x) {
  uint32_t r;
  asm("cvt.rn.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}
// two fp32 lanes per instruction (packed f32x2 arithmetic, round to nearest even, the
// same results as two scalar operations)
__device__ __forceinline__ void mul2(float &a0, float &a1, float b0, float b1) {
  asm("{\n\t.reg .b64 x, y;\n\tmov.b64 x, {%0, %1};\n\tmov.b64 y, {%2, %3};\n\t"
      "mul.rn.f32x2 x, x, y;\n\tmov.b64 {%0, %1}, x;\n\t}"
      : "+f"(a0), "+f"(a1) : "f"(b0), "f"(b1));
}
__device__ __forceinline__ void sub2(float &a0, float &a1, float b0, float b1) {
  asm("{\n\t.reg .b64 x, y;\n\tmov.b64 x, {%0, %1};\n\tmov.b64 y, {%2, %3};\n\t"
      "sub.rn.f32x2 x, x, y;\n\tmov.b64 {%0, %1}, x;\n\t}"
      : "+f"(a0), "+f"(a1) : "f"(b0), "f"(b1));
}
__device__ __forceinline__ void fma2(float &a0, float &a1, float b0, float b1, float c0, float c1) {
  asm("{\n\t.reg .b64 x, y, z;\n\tmov.b64 x, {%0, %1};\n\tmov.b64 y, {%2, %3};\n\t"
      "mov.b64 z, {%4, %5};\n\tfma.rn.f32x2 x, y, z, x;\n\tmov.b64 {%0, %1}, x;\n\t}"
      : "+f"(a0), "+f"(a1) : "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}
__device__ __forceinline__ void ld8f(const float *p, float *x) {
  const float4 a = reinterpret_cast<const float4 *>(p)[0];
  const float4 b = reinterpret_cast<const float4 *>(p)[1];
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}
// eight operand values as two 16-byte shared-memory stores (see st_shared_f4)
__device__ __forceinline__ void st8f(unsigned char *base, uint32_t off_lo, uint32_t off_hi,
                                     const float *y) {
  st_shared_f4(base + off_lo, y[0], y[1], y[2], y[3]);
  st_shared_f4(base + off_hi, y[4], y[5], y[6], y[7]);
}

#ifdef KDA_PHASE_PROFILE
// Cycles per step of the loops, summed over every CTA (profiling builds only):
// group A (thread 0): 0 wait for O^T/Y^T(m-1), 1 wait for the tiles of chunk m+1,
// 2 gate(m+1), 3 rows(m), 4 wait for A|P(m), 5 read, 7 solve up to the diagonal blocks,
// 6 the rest of the solve; group B (thread 256): 8 wait for O^T/Y^T(n), 9 scale, 10 wait
// for the next gate, 11 Khat^T, 12 wait for the last products, 13 out, 14 V^T.
// Entry 15 counts the chunks.
__device__ unsigned long long g_phase_cycles[16];
#define KDA_PHASE(k)                                              \
  do {                                                            \
    if (prof) {                                                   \
      const long long now_ = clock64();                           \
      phase_acc[k] += (unsigned long long)(now_ - phase_t);       \
      phase_t = now_;                                             \
    }                                                             \
  } while (0)
#else
#define KDA_PHASE(k) \
  do {               \
  } while (0)
#endif

// LOGITS: the gate arrives as bf16 logits (fused gate activation) instead of fp32 g.
// LOCAL: the local state of a segment (context-parallel pass 1): S_loc from a zero state
// with the segment's values, and, in the same pass over the chunks, the transition M
// from the identity with zero values (the augmented columns [V | 0] from [0 | I]), both
// sharing the chunk's gate, row operands, A, T and Khat.  M^T lives in TMEM columns the
// local state leaves free: Y_M^T where O^T would be, U_M^T over Y_S^T once U_S^T has
// read it.
template <typename TOut, bool LOGITS, bool LOCAL>
__global__ void __launch_bounds__(NT + 64, 1)
    prefill_tc_kernel(const PrefillParams p, const __grid_constant__ TcMaps maps) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char *sm = align1024_shared(smem_raw);
  float *NS = reinterpret_cast<float *>(sm + OFF_NS);
  float *TS = reinterpret_cast<float *>(sm + OFF_TS);
  float *XS = reinterpret_cast<float *>(sm + OFF_XS);
  float *GC = reinterpret_cast<float *>(sm + OFF_GC);
  float *BT = reinterpret_cast<float *>(sm + OFF_BT);
  uint64_t *bars = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
  uint64_t *bar_tma = bars + 0;   // [2] TMA -> group A: raw buffer b landed
  uint64_t *bar_ap = bars + 2;    // commit: A|P products done
  uint64_t *bar_oy = bars + 3;    // commit: O^T and Y^T products done (S^T read)
  uint64_t *bar_u = bars + 4;     // commit: U^T product done (control only)
  uint64_t *bar_fin = bars + 5;   // commit: the chunk's last products done
  uint64_t *ops_ap = bars + 6;    // group A -> control: A|P operands built
  uint64_t *raw_free = bars + 7;  // A and B -> control: a raw buffer fully read
  uint64_t *ops_oy = bars + 8;    // A (gamma*Q) and B (gamma*K, V^T) -> control
  uint64_t *ops_tb = bars + 9;    // group A -> control: T Diag(beta) ready
  uint64_t *ops_sc = bars + 10;   // group B -> control: S^T scaled by gamma_31
  uint64_t *gate_ok = bars + 11;  // [2] group A -> group B: cumulative gate of a chunk ready
  uint64_t *bar_us = bars + 13;   // local state: commit of U_S^T (before U_M^T overwrites Y_S^T)
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(bars + 14);
  volatile int *s_abort = reinterpret_cast<volatile int *>(s_tmem + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane_id = tid & 31;
  const bool control = warp >= NT / 32;            // warps 16, 17: TMA and MMA issue
  const bool group_a = warp < NA / 32;
  const int qd = warp & 3;                         // TMEM lane quarter of a worker warp
  const int cg = (warp >> 2) & 1;                  // its half of the columns / tokens
  const int l = 32 * qd + lane_id;                 // its TMEM lane / channel
  const uint32_t lane_base = (uint32_t)(32 * qd) << 16;
  const int H = p.H;
  // one CTA per (request or segment, head)
  const int pairs = p.n_req * H;
  const int rem = (int)(blockIdx.x % pairs);
  const int r = p.order ? p.order[rem / H] : rem / H;
  const int h = rem % H;
  // q, P and O only where o is written: not in the local-state pass, nor in a run that
  // only wants states (the backward's recompute).  A runtime flag keeps the register
  // allocation tight.
  const bool has_q = !p.local_mode && p.o != nullptr;
  const uint64_t wait_ns = p.wait_ns ? p.wait_ns : 2000000000ull;
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
    mbar_init(bar_tma + 1, 1);
    mbar_init(bar_ap, 1);
    mbar_init(bar_oy, 1);
    mbar_init(bar_u, 1);
    mbar_init(bar_fin, 1);
    mbar_init(ops_ap, NA / 32);
    mbar_init(raw_free, NT / 32);
    mbar_init(ops_oy, NT / 32);
    mbar_init(ops_tb, NA / 32);
    mbar_init(ops_sc, (NT - NA) / 32);
    mbar_init(gate_ok, NA / 32);
    mbar_init(gate_ok + 1, NA / 32);
    mbar_init(bar_us, 1);
    *s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = *s_tmem;
  const int n_chunks = (len + C - 1) / C;

  // What each issuing thread of the control warp issued, so that a CTA that gives up
  // can let it land: the TMA loads per raw buffer, and the barrier and phase parity of
  // the thread's last commit (a commit covers every earlier product of its thread).
  uint32_t tma_n0 = 0u, tma_n1 = 0u;
  uint64_t *last_bar = nullptr;
  uint32_t last_par = 0u;

#ifdef KDA_PHASE_PROFILE
  // thread 0's (group A) and thread 256's (group B) per-step sums, in spare bytes
  const bool prof = tid == 0 || tid == NA;
  unsigned long long *phase_acc = reinterpret_cast<unsigned long long *>(sm + OFF_BAR + 128);
  if (tid == 0)
    for (int k = 0; k < 16; ++k) phase_acc[k] = 0ull;
  __syncthreads();
  long long phase_t = clock64();
#endif

  // One arrival per warp.  warp_arrive hands shared-memory operands to the tensor
  // cores, so its lanes' generic writes are first made visible to the async proxy;
  // warp_signal orders only ordinary shared-memory and TMEM accesses (the arrival's
  // release and the waiter's acquire), as for tables read by other warps, tiles
  // that were only read, and TMEM written with tcgen05.st.
  auto warp_signal = [&](uint64_t *bar) {
    tc_fence_before();
    __syncwarp();
    if (lane_id == 0) mbar_arrive(bar);
  };
  auto warp_arrive = [&](uint64_t *bar) {
    fence_async_smem();
    warp_signal(bar);
  };

  if (control) {
    // ==================== control warp: TMA and MMA issue ====================
    // Two threads in two warps issue independently, so that neither group's products
    // wait for the other's (and a waiting thread never holds up the other's warp):
    // warp 16 the TMA loads, A|P and U^T (group A's chain), warp 17 O^T, Y^T and the
    // last products (the state chain).  Products of the two threads that depend on
    // each other are ordered by the barriers below: U^T(m) waits for O^T, Y^T(m)
    // (whose commit also covers warp 17's earlier products of chunk m-1), the last
    // products of chunk m for U^T(m).
    if (lane_id == 0) {
      tma_prefetch_desc(&maps.q);
      tma_prefetch_desc(&maps.k);
      tma_prefetch_desc(&maps.v);
      tma_prefetch_desc(&maps.g);
      const uint32_t tx = (has_q ? 3u : 2u) * 8192u + (LOGITS ? 8192u : 16384u);
      auto issue_tma = [&](int m) {
        const int b = m & 1;
        unsigned char *raw = sm + OFF_RAW + b * RAW_BYTES;
        mbar_expect_tx(bar_tma + b, tx);
        const int y = bos + m * C;
        for (int half = 0; half < 2; ++half) {
          const int x = h * DH + 64 * half;
          tma_load_2d(raw + R_K + 4096 * half, &maps.k, x, y, bar_tma + b);
          if (has_q) tma_load_2d(raw + R_Q + 4096 * half, &maps.q, x, y, bar_tma + b);
          tma_load_2d(raw + R_V + 4096 * half, &maps.v, x, y, bar_tma + b);
        }
        if (LOGITS) {
          for (int half = 0; half < 2; ++half)
            tma_load_2d(raw + R_G + 4096 * half, &maps.g, h * DH + 64 * half, y, bar_tma + b);
        } else {
          for (int q4 = 0; q4 < 4; ++q4)
            tma_load_2d(raw + R_G + 4096 * q4, &maps.g, h * DH + 32 * q4, y, bar_tma + b);
        }
        if (b) ++tma_n1; else ++tma_n0;
      };
      // one commit per chunk on each barrier: phase m of a barrier belongs to chunk m
      auto commit = [&](uint64_t *bar, int m) {
        mma_commit(bar);
        last_bar = bar;
        last_par = (uint32_t)m & 1u;
      };
      uint32_t ph_ops_ap = 0, ph_raw = 0, ph_ops_oy = 0, ph_tb = 0, ph_sc = 0, ph_oy = 0,
               ph_u = 0;
      auto cwait = [&](uint64_t *bar, uint32_t &ph) -> bool {
        const bool good = *s_abort == 0 && mbar_wait_ni(bar, ph, wait_ns, s_abort);
        ph ^= 1u;
        if (!good) {
          *s_abort = 1;
          set_status(p.status, STATUS_TIMEOUT);
        }
        tc_fence_after();
        return good;
      };
      // A | P: [L_k ; L_q] R'^T, N = 32 over the 128 key channels
      auto mma_ap = [&](int m) {
        const uint32_t rp = smem_u32(sm + OFF_RP);
        const uint32_t id = idesc_tf32(C);
#pragma unroll
        for (int s = 0; s < DH / 8; ++s)
          mma_tf32_ts(tm + TM_AP, tm + TM_L + 8 * s, sw128_desc(rp, C, s), id, s > 0);
        commit(bar_ap, m);
      };
      // O^T = S^T (gamma Q)^T and Y^T = V^T - S^T (gamma K)^T
      auto mma_oy = [&](int m) {
        const uint32_t id = idesc_tf32(C), idn = idesc_tf32(C, true);
        const uint32_t gq = smem_u32(sm + OFF_GQ), gk = smem_u32(sm + OFF_GK);
#pragma unroll
        for (int s = 0; s < DH / 8; ++s) {
          if (has_q) mma_tf32_ts(tm + TM_O, tm + TM_S + 8 * s, sw128_desc(gq, C, s), id, s > 0);
          mma_tf32_ts(tm + TM_Y, tm + TM_S + 8 * s, sw128_desc(gk, C, s), idn, true);
          // local state: Y_M^T = -M^T (gamma K)^T (zero values)
          if (LOCAL) mma_tf32_ts(tm + TM_O, tm + TM_M + 8 * s, sw128_desc(gk, C, s), idn, s > 0);
        }
        commit(bar_oy, m);
      };
      // U^T = Y^T (T Diag(beta))^T; local state: then U_M^T = Y_M^T (T Diag(beta))^T over
      // Y_S^T, once U_S^T is done reading it
      uint32_t ph_us = 0;
      auto mma_u = [&](int m) -> bool {
        const uint32_t tb = smem_u32(sm + tb_off(m));
        const uint32_t id = idesc_tf32(C);
#pragma unroll
        for (int s = 0; s < C / 8; ++s)
          mma_tf32_ts(tm + TM_U, tm + TM_Y + 8 * s, sw128_desc(tb, C, s), id, s > 0);
        if constexpr (LOCAL) {
          commit(bar_us, m);
          if (!cwait(bar_us, ph_us)) return false;
#pragma unroll
          for (int s = 0; s < C / 8; ++s)
            mma_tf32_ts(tm + TM_Y, tm + TM_O + 8 * s, sw128_desc(tb, C, s), id, s > 0);
        }
        commit(bar_u, m);
        return true;
      };
      // O^T += U^T P^T and S^T += U^T Khat (S^T already scaled by gamma_31)
      auto mma_fin = [&](int m) {
        const uint32_t pp = smem_u32(sm + pp_off(m)), kh = smem_u32(sm + kh_off(m));
        const uint32_t id32 = idesc_tf32(C), id128 = idesc_tf32(DH);
#pragma unroll
        for (int s = 0; s < C / 8; ++s) {
          if (has_q) mma_tf32_ts(tm + TM_O, tm + TM_U + 8 * s, sw128_desc(pp, C, s), id32, true);
          mma_tf32_ts(tm + TM_S, tm + TM_U + 8 * s, sw128_desc(kh, DH, s), id128, true);
          // local state: M^T += U_M^T Khat
          if (LOCAL) mma_tf32_ts(tm + TM_M, tm + TM_Y + 8 * s, sw128_desc(kh, DH, s), id128, true);
        }
        commit(bar_fin, m);
      };
      if (warp == NT / 32) {
        if (n_chunks > 0) issue_tma(0);
        if (n_chunks > 1) issue_tma(1);
        for (int m = 0; m < n_chunks; ++m) {
          if (!cwait(ops_ap, ph_ops_ap)) break;
          mma_ap(m);
          // chunk m's tiles are read (group A signs with the A|P operands, group B with
          // V^T(m), a chunk earlier): chunk m + 2 may load, a whole chunk before its gate
          if (!cwait(raw_free, ph_raw)) break;
          if (m + 2 < n_chunks) issue_tma(m + 2);
          if (!cwait(ops_tb, ph_tb)) break;
          if (!cwait(bar_oy, ph_oy)) break;  // Y^T is U^T's A operand
          if (!mma_u(m)) break;
        }
      } else {
        for (int m = 0; m < n_chunks; ++m) {
          if (!cwait(ops_oy, ph_ops_oy)) break;
          mma_oy(m);
          if (!cwait(ops_sc, ph_sc)) break;
          if (!cwait(bar_u, ph_u)) break;  // U^T is the A operand of the last products
          mma_fin(m);
        }
      }
    }
  } else if (group_a) {
    // ============ group A (warps 0-7): gate, row operands, read-out, solve ============
    uint32_t ph_tma = 0u, ph_ap = 0, ph_oy = 0;  // ph_tma: bit b for buffer b
    auto wsync = [&]() { named_sync(1, NA); };
    // every thread waits, and the vote at the group's named barrier gives every thread
    // the outcome, so that an abort is taken by all together
    auto wwait = [&](uint64_t *bar, uint32_t &ph) -> bool {
      const bool got = mbar_wait_ni(bar, ph, wait_ns, s_abort);
      ph ^= 1u;
      const bool bad = named_sync_or(1, NA, !got || *s_abort != 0);
      if (bad) {
        if (!got) set_status(p.status, STATUS_TIMEOUT);
        *s_abort = 1;
      }
      tc_fence_after();
      return !bad;
    };
    auto wait_tma = [&](int m) -> bool {
      uint32_t ph = (ph_tma >> (m & 1)) & 1u;
      const bool got = wwait(bar_tma + (m & 1), ph);
      ph_tma ^= 1u << (m & 1);
      return got;
    };
    // T Diag(beta) is lower triangular: its block above the diagonal stays zero
    if (tid < 128)
      *reinterpret_cast<float4 *>(sm + tb_off(tid >> 6) +
                                  sw128_chunk(C, (tid >> 2) & 15, 16 + 4 * (tid & 3))) =
          make_float4(0.f, 0.f, 0.f, 0.f);

    // beta of chunk m, row tid (warp 0), loaded a chunk ahead and checked when stored;
    // a predicated load, so that nothing waits for it before its use a chunk later
    auto load_beta = [&](int m) -> float {
      const int t = m * C + tid;
      const bool in = tid < C && m < n_chunks && t < len;
      const float *src = p.beta + (in ? (size_t)(bos + t) * H + h : 0);
      float b = 0.f;
      asm volatile(
          "{\n\t.reg .pred q;\n\tsetp.ne.u32 q, %2, 0;\n\t@q ld.global.nc.f32 %0, [%1];\n\t}"
          : "+f"(b)
          : "l"(src), "r"((uint32_t)in));
      return b;
    };
    float beta_pref = load_beta(0);

    // ---- gate(m): cumulative gate (thread = key channel gc, tokens 16 gh .. 16 gh + 15:
    // the two halves of a channel sit in one warp, lanes 16 apart) ----
    const int gc = 16 * warp + (lane_id & 15), gh = lane_id >> 4;
    auto w_gate = [&](int m) {
      const int nr = min(C, len - m * C);
      unsigned char *raw = sm + OFF_RAW + (m & 1) * RAW_BYTES;
      if (tid < C) {
        if (p.validate && !(beta_pref >= 0.f && beta_pref <= 1.f))
          set_status(p.status, STATUS_GATE_RANGE);
        BT[(m & 1) * C + tid] = beta_pref;
      }
      beta_pref = load_beta(m + 1);
      // every row of the tile is loaded (rows past the chunk's end hold other data or the
      // zero fill) and masked afterwards, so that the 16 loads issue back to back
      float gv[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int t = 16 * gh + j;
        gv[j] = LOGITS ? gate_from_logit(bf16_at(raw + R_G, t, gc))
                       : *reinterpret_cast<const float *>(raw + R_G + f32_off(t, gc));
      }
#pragma unroll
      for (int j = 0; j < 16; ++j) gv[j] = (16 * gh + j < nr) ? gv[j] : 0.f;
      if (!LOGITS && p.validate) {
        bool bad = false;
#pragma unroll
        for (int j = 0; j < 16; ++j) bad |= !(gv[j] >= kGateLower && gv[j] <= 0.f);
        if (bad) set_status(p.status, STATUS_GATE_RANGE);
      }
#pragma unroll
      for (int j = 1; j < 16; ++j) gv[j] += gv[j - 1];
      const float first = __shfl_sync(0xffffffffu, gv[15], lane_id & 15);
      const float off = gh ? first : 0.f;
      float *gtab = reinterpret_cast<float *>(sm + OFF_GT + (m & 1) * GT_BYTES) +
                    16 * gh * LDG + gc;
#pragma unroll
      for (int j = 0; j < 16; ++j) gtab[j * LDG] = (gv[j] + off) * LOG2E;
      if (gh) GC[(m & 3) * DH + gc] = ex2((gv[15] + off) * LOG2E);
      warp_signal(gate_ok + (m & 1));
    };

    // ---- rows(m): the row operands (thread = row i, channels 64 cg .. 64 cg + 63) ----
    // lane quarter 0: L_k = k exp(G_i - G_15) -> TMEM lanes 0-31
    // lane quarter 1: L_q = q exp(G_i - G_15) -> TMEM lanes 32-63
    // lane quarter 2: R'  = k exp(G_15 - G_i) -> smem
    // lane quarter 3: gamma*Q = q exp(G_i)    -> smem  (gamma*K: group B, with Khat^T)
    // (one straight-line loop per quarter, so that loads issue ahead of the stores)
    auto w_rows = [&](int m) {
      const int nr = min(C, len - m * C);
      const unsigned char *raw = sm + OFF_RAW + (m & 1) * RAW_BYTES;
      const int i = lane_id;
      const bool valid = i < nr;
      const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
      const float *gt = reinterpret_cast<const float *>(sm + OFF_GT + (m & 1) * GT_BYTES);
      auto load_x = [&](uint32_t tile, int c) {
        return valid ? *reinterpret_cast<const uint4 *>(raw + tile + bf16_chunk(i, c)) : z4;
      };
      if (qd <= 1) {  // L = x exp(G_i - G_15) -> TMEM lanes 32 qd + i
        if (qd == 1 && !has_q) return;
        const uint32_t tile = qd == 0 ? R_K : R_Q;
#pragma unroll 1
        for (int jj = 0; jj < 8; ++jj) {
          const int c = 64 * cg + 8 * jj;
          float x[8], g[8], gr[8];
          bf16_x8(load_x(tile, c), x);
          ld8g(gt, i, c, g);
          ld8g(gt, MREF, c, gr);
#pragma unroll
          for (int e = 0; e < 8; e += 2) sub2(g[e], g[e + 1], gr[e], gr[e + 1]);
#pragma unroll
          for (int e = 0; e < 8; ++e) g[e] = ex2(g[e]);
#pragma unroll
          for (int e = 0; e < 8; e += 2) mul2(x[e], x[e + 1], g[e], g[e + 1]);
#pragma unroll
          for (int e = 0; e < 8; ++e) x[e] = tf32_rn(x[e]);
          tmem_st8(tm + lane_base + TM_L + c, x);
        }
        tmem_wait_st();
      } else if (qd == 2) {  // R' = k exp(G_15 - G_i)
#pragma unroll 1
        for (int jj = 0; jj < 8; ++jj) {
          const int c = 64 * cg + 8 * jj;
          float x[8], g[8], gr[8];
          bf16_x8(load_x(R_K, c), x);
          ld8g(gt, i, c, g);
          ld8g(gt, MREF, c, gr);
#pragma unroll
          for (int e = 0; e < 8; e += 2) sub2(gr[e], gr[e + 1], g[e], g[e + 1]);
#pragma unroll
          for (int e = 0; e < 8; ++e) gr[e] = ex2(gr[e]);
#pragma unroll
          for (int e = 0; e < 8; e += 2) mul2(x[e], x[e + 1], gr[e], gr[e + 1]);
#pragma unroll
          for (int e = 0; e < 8; ++e) x[e] = tf32_rn(x[e]);
          st8f(sm + OFF_RP, sw128_chunk(C, i, c), sw128_chunk(C, i, c + 4), x);
        }
      } else if (has_q) {  // gamma*Q = q exp(G_i)
#pragma unroll 1
        for (int jj = 0; jj < 8; ++jj) {
          const int c = 64 * cg + 8 * jj;
          float x[8], g[8];
          bf16_x8(load_x(R_Q, c), x);
          ld8g(gt, i, c, g);
#pragma unroll
          for (int e = 0; e < 8; ++e) g[e] = ex2(g[e]);
#pragma unroll
          for (int e = 0; e < 8; e += 2) mul2(x[e], x[e + 1], g[e], g[e + 1]);
#pragma unroll
          for (int e = 0; e < 8; ++e) x[e] = tf32_rn(x[e]);
          st8f(sm + OFF_GQ, sw128_chunk(C, i, c), sw128_chunk(C, i, c + 4), x);
        }
      }
    };

    // ---- read(m): Diag(beta) A and P out of TMEM (after the A|P products) ----
    auto w_read = [&](int m) {
      const int i = lane_id;
      if (qd == 0) {  // row i of A, columns 16 cg ..: N = beta_i A_ij for j < i
        float a[16];
        tmem_ld16(tm + lane_base + TM_AP + 16 * cg, a);
        tmem_wait_ld();
        const float bi = BT[(m & 1) * C + i];
#pragma unroll
        for (int e = 0; e < 16; ++e) a[e] = (16 * cg + e < i) ? bi * a[e] : 0.f;
        float4 *nd = reinterpret_cast<float4 *>(NS + i * LDN + 16 * cg);
#pragma unroll
        for (int e = 0; e < 4; ++e) nd[e] = make_float4(a[4 * e], a[4 * e + 1], a[4 * e + 2], a[4 * e + 3]);
      } else if (qd == 1 && has_q) {  // row i of P, inclusive lower, tf32 B operand
        float a[16];
        tmem_ld16(tm + lane_base + TM_AP + 16 * cg, a);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) a[e] = (16 * cg + e <= i) ? tf32_rn(a[e]) : 0.f;
        unsigned char *pp = sm + pp_off(m);
        st8f(pp, sw128_chunk(C, i, 16 * cg), sw128_chunk(C, i, 16 * cg + 4), a);
        st8f(pp, sw128_chunk(C, i, 16 * cg + 8), sw128_chunk(C, i, 16 * cg + 12), a + 8);
      }
    };

    // ---- solve(m): T = (I + Diag(beta) A)^-1 by 16 x 16 blocks, then T Diag(beta) ----
    auto w_solve = [&](int m) {
      unsigned char *tb = sm + tb_off(m);
      wsync();  // Diag(beta) A complete
      if (warp == 2) {
        // the two diagonal blocks, row by row: t_i = e_i - sum_{j<i} N_ij t_j, one
        // column per lane (lanes 0-15: block 0, lanes 16-31: block 1); the sum runs
        // in two halves to shorten the dependent chain
        const int o = 16 * (lane_id >> 4), c = lane_id & 15;
        float t[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float4 *nrow = reinterpret_cast<const float4 *>(NS + (o + i) * LDN + o);
          float acc0 = (i == c) ? 1.f : 0.f, acc1 = 0.f;
#pragma unroll
          for (int j4 = 0; j4 < 4; ++j4) {
            if (4 * j4 >= i) break;
            const float4 n4 = nrow[j4];
            const float nv[4] = {n4.x, n4.y, n4.z, n4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int j = 4 * j4 + e;
              if (j < i) {
                if (j & 1) acc1 -= nv[e] * t[j];
                else acc0 -= nv[e] * t[j];
              }
            }
          }
          t[i] = acc0 + acc1;
        }
        const float bc = BT[(m & 1) * C + o + c];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          TS[(o + i) * LDN + o + c] = t[i];
          st_shared_f1(tb + sw128_offset(C, o + i, o + c), tf32_rn(t[i] * bc));
        }
      }
      wsync();  // diagonal blocks ready
      KDA_PHASE(7);
      {  // T10 = -T11 (N10 T00): one element (i, c) per thread of the group
        // the T00 entries above the diagonal and the T11 entries past row i are zero, so
        // the sums run over all 16 terms without branches, in two halves each
        const int i = tid >> 4, c = tid & 15;
        float x0 = 0.f, x1 = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j)
          fma2(x0, x1, NS[(16 + i) * LDN + j], NS[(16 + i) * LDN + 8 + j], TS[j * LDN + c],
               TS[(8 + j) * LDN + c]);
        XS[i * LDX + c] = x0 + x1;
        wsync();
        float y0 = 0.f, y1 = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j)
          fma2(y0, y1, TS[(16 + i) * LDN + 16 + j], TS[(16 + i) * LDN + 24 + j], XS[j * LDX + c],
               XS[(8 + j) * LDX + c]);
        st_shared_f1(tb + sw128_offset(C, 16 + i, c), tf32_rn(-(y0 + y1) * BT[(m & 1) * C + c]));
      }
    };

    // The gate of chunk m+1 runs while the A|P products of chunk m do (its table sits in
    // chunk m+1's own raw buffer, which group B has read for chunk m-1 before the tiles
    // of chunk m+1 could load).  Its barrier is one of a pair, by chunk parity, so group
    // A may finish a gate before group B has taken the previous one.
    bool ok = true;
    if (n_chunks > 0 && (ok = wait_tma(0))) {
      w_gate(0);
      wsync();  // every warp's channels of the table before any row operand reads them
    }
    for (int m = 0; ok && m < n_chunks; ++m) {
      // chunk m-1's O^T and Y^T products are done: gamma*Q/K are free (and, through
      // group B, chunk m-2's last products are done too)
      if (m > 0 && !(ok = wwait(bar_oy, ph_oy))) break;
      KDA_PHASE(0);
      w_rows(m);
      warp_signal(raw_free);
      warp_arrive(ops_ap);
      warp_signal(ops_oy);  // gamma*Q made visible by the fence of the arrival above
      KDA_PHASE(3);
      if (m + 1 < n_chunks) {
        if (!(ok = wait_tma(m + 1))) break;
        KDA_PHASE(1);
        w_gate(m + 1);
        KDA_PHASE(2);
      }
      if (!(ok = wwait(bar_ap, ph_ap))) break;
      KDA_PHASE(4);
      w_read(m);  // P reaches the tensor cores after the solve's arrival (fence there)
      KDA_PHASE(5);
      w_solve(m);
      warp_arrive(ops_tb);
      KDA_PHASE(6);
    }
  } else {
    // ====== group B (warps 8-15): state scaling, Khat^T, outputs, V^T, states ======
    uint32_t ph_oy = 0, ph_fin = 0;
    // every thread waits, and the vote at the group's named barrier gives every thread
    // the outcome, so that an abort is taken by all together
    auto bwait = [&](uint64_t *bar, uint32_t &ph) -> bool {
      const bool got = mbar_wait_ni(bar, ph, wait_ns, s_abort);
      ph ^= 1u;
      const bool bad = named_sync_or(2, NT - NA, !got || *s_abort != 0);
      if (bad) {
        if (!got) set_status(p.status, STATUS_TIMEOUT);
        *s_abort = 1;
      }
      tc_fence_after();
      return !bad;
    };
    const int w8 = warp - NA / 32;  // 0..7

    // initial state -> S^T in TMEM (lane v holds S[:, v]), columns 64 cg ..
    {
      const float *s0 =
          p.initial_state ? p.initial_state + ((size_t)(r * H + h)) * DH * DH : nullptr;
#pragma unroll 1
      for (int q8 = 0; q8 < 8; ++q8) {
        const int c0 = 64 * cg + 8 * q8;
        float v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = (!LOCAL && s0) ? s0[(size_t)(c0 + j) * DH + l] : 0.f;
        tmem_st8(tm + lane_base + TM_S + c0, v);
        if constexpr (LOCAL) {  // M^T = I
#pragma unroll
          for (int j = 0; j < 8; ++j) v[j] = c0 + j == l ? 1.f : 0.f;
          tmem_st8(tm + lane_base + TM_M + c0, v);
        }
      }
      tmem_wait_st();
    }

    // ---- scale(n): S^T <- S^T Diag(gamma_31) once the O^T and Y^T products read S^T ----
    auto w_scale = [&](int n) {
      const float *gc = GC + (n & 3) * DH;
      auto scale_cols = [&](uint32_t base) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int c0 = 64 * cg + 16 * q;
          float v[16];
          tmem_ld16(tm + lane_base + base + c0, v);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; j += 8) {
            float f[8];
            ld8f(gc + c0 + j, f);
#pragma unroll
            for (int e = 0; e < 8; e += 2) mul2(v[j + e], v[j + e + 1], f[e], f[e + 1]);
          }
          tmem_st16(tm + lane_base + base + c0, v);
        }
      };
      scale_cols(TM_S);
      if constexpr (LOCAL) scale_cols(TM_M);  // the transition scales like the state
      tmem_wait_st();
    };

    // ---- khat(m): Khat^T = (k exp(G_31 - G))^T and gamma*K = k exp(G), one pass over k
    // (thread = row i, channels 16 w8 ..); gamma*K's tile is free once O^T, Y^T(m-1)
    // are done, which precedes this ----
    auto w_khat = [&](int m) {
      const int nr = min(C, len - m * C);
      const unsigned char *raw = sm + OFF_RAW + (m & 1) * RAW_BYTES;
      const float *gtab = reinterpret_cast<const float *>(sm + OFF_GT + (m & 1) * GT_BYTES);
      const int i = lane_id;
      // element (channel c + e, token i) of the Khat^T tile: row c + e, 16-byte chunk
      // (i >> 2) ^ e (c % 8 == 0), so eight offsets serve both channel groups
      unsigned char *kh = sm + kh_off(m) + (i & 3) * 4;
      uint32_t koff[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) koff[e] = e * 128 + (((i >> 2) ^ e) << 4);
#pragma unroll 1  // rolled: smaller code (see mbar_wait_slow)
      for (int u = 0; u < 2; ++u) {
        const int c = 16 * w8 + 8 * u;
        float x[8], g[8], ge[8], gk[8];
        bf16_x8(i < nr ? *reinterpret_cast<const uint4 *>(raw + R_K + bf16_chunk(i, c))
                       : make_uint4(0u, 0u, 0u, 0u),
                x);
        ld8g(gtab, i, c, g);
        ld8g(gtab, C - 1, c, ge);
#pragma unroll
        for (int e = 0; e < 8; e += 2) sub2(ge[e], ge[e + 1], g[e], g[e + 1]);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          ge[e] = ex2(ge[e]);
          gk[e] = ex2(g[e]);
        }
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
          mul2(ge[e], ge[e + 1], x[e], x[e + 1]);
          mul2(gk[e], gk[e + 1], x[e], x[e + 1]);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          st_shared_f1(kh + c * 128 + koff[e], tf32_rn(ge[e]));
          gk[e] = tf32_rn(gk[e]);
        }
        st8f(sm + OFF_GK, sw128_chunk(C, i, c), sw128_chunk(C, i, c + 4), gk);
      }
    };

    // ---- out(n): O^T -> o (lane = value channel, tokens 16 cg ..), snapshot ----
    auto w_out = [&](int n) {
      const int c0 = n * C, nr = min(C, len - c0);
      if (go) {
        float o16[16];
        tmem_ld16(tm + lane_base + TM_O + 16 * cg, o16);
        tmem_wait_ld();
        // one pointer stepped by a token's row (64-bit index arithmetic per store was a
        // large part of this step, which lies on the state chain)
        TOut *dst = go + ((size_t)(bos + c0 + 16 * cg) * H + h) * DH + l;
        const size_t step = (size_t)H * DH;
        const int nt = nr - 16 * cg;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          if (j < nt) store_elem(dst, 0, o16[j]);
          dst += step;
        }
      }
      if (snaps_ok && nr == C && (c0 + C) % p.snapshot_stride == 0) {
        const size_t row = (size_t)p.cu_snapshots[r] + (c0 + C) / p.snapshot_stride - 1;
        float *dst = p.snapshots + (row * H + h) * (size_t)DH * DH;
#pragma unroll 1
        for (int q8 = 0; q8 < 8; ++q8) {
          const int k0 = 64 * cg + 8 * q8;
          float v[8];
          tmem_ld8(tm + lane_base + TM_S + k0, v);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 8; ++j) dst[(size_t)(k0 + j) * DH + l] = v[j];
        }
      }
    };

    // ---- vt(m): V^T -> TMEM (lane = value channel, tokens 16 cg ..) ----
    auto w_vt = [&](int m) {
      const int nr = min(C, len - m * C);
      // row t = 16 cg + j of the swizzled v tile: the 16-byte chunk of channel l sits at
      // chunk index ((l & 63) >> 3) ^ (j & 7), so eight offsets serve all sixteen rows
      const unsigned char *row0 = sm + OFF_RAW + (m & 1) * RAW_BYTES + R_V + (l >> 6) * 4096 +
                                  16 * cg * 128 + (l & 7) * 2;
      const int c8 = (l & 63) >> 3, nv = nr - 16 * cg;
      float v16[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const unsigned short u =
            *reinterpret_cast<const unsigned short *>(row0 + j * 128 + ((c8 ^ (j & 7)) << 4));
        v16[j] = j < nv ? bf16_lo(u) : 0.f;
      }
      tmem_st16(tm + lane_base + TM_Y + 16 * cg, v16);
      tmem_wait_st();
    };

    bool ok = true;
    if (n_chunks > 0) {
      uint32_t ph = 0;
      if ((ok = bwait(gate_ok, ph))) {
        w_khat(0);
        w_vt(0);
        warp_signal(raw_free);
        warp_arrive(ops_oy);
      }
    }
    for (int n = 0; ok && n < n_chunks; ++n) {
      const bool more = n + 1 < n_chunks;
      if (!(ok = bwait(bar_oy, ph_oy))) break;
      KDA_PHASE(8);
      w_scale(n);
      warp_signal(ops_sc);
      KDA_PHASE(9);
      if (more) {
        uint32_t ph = ((n + 1) >> 1) & 1u;
        if (!(ok = bwait(gate_ok + ((n + 1) & 1), ph))) break;
        KDA_PHASE(10);
        w_khat(n + 1);  // the other Khat^T buffer: chunk n-1's last products are done
        KDA_PHASE(11);
      }
      if (!(ok = bwait(bar_fin, ph_fin))) break;
      KDA_PHASE(12);
      w_out(n);
      KDA_PHASE(13);
      if (more) {
        w_vt(n + 1);
        warp_signal(raw_free);  // before ops_oy: group A's next arrivals wait for it
        warp_arrive(ops_oy);
      }
      KDA_PHASE(14);
    }

    // the final state (local state: S_loc and the transition M)
    auto write_state = [&](float *dst_base, uint32_t col) {
      float *dst = dst_base + ((size_t)(r * H + h)) * DH * DH;
#pragma unroll 1
      for (int q8 = 0; q8 < 8; ++q8) {
        const int k0 = 64 * cg + 8 * q8;
        float v[8];
        tmem_ld8(tm + lane_base + col + k0, v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 8; ++j) dst[(size_t)(k0 + j) * DH + l] = v[j];
      }
    };
    float *fin = LOCAL ? p.s_loc : p.final_state;
    if (ok && fin) {
      tc_fence_after();
      write_state(fin, TM_S);
      if constexpr (LOCAL) write_state(p.m, TM_M);
    }
  }
#ifdef KDA_PHASE_PROFILE
  if (tid == 0) atomicAdd(&g_phase_cycles[15], (unsigned long long)n_chunks);
  __syncthreads();
  if (tid == 0)
    for (int k = 0; k < 15; ++k) atomicAdd(&g_phase_cycles[k], phase_acc[k]);
#endif

  tc_fence_before();
  __syncthreads();
  if (*s_abort && control && lane_id == 0) {
    // the CTA gave up: let the copies and products it issued land before it releases
    // its shared and tensor memory (at most one load per buffer and, the products of
    // a thread completing in order, its last commit are outstanding)
    if (tma_n0) mbar_wait(bar_tma, (tma_n0 - 1u) & 1u, 100000000ull);
    if (tma_n1) mbar_wait(bar_tma + 1, (tma_n1 - 1u) & 1u, 100000000ull);
    if (last_bar) mbar_wait(last_bar, last_par, 100000000ull);
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

// A [rows, inner] row-major tensor read as boxes of [C rows, box_inner elements]
// (box_inner * esize = 128 bytes, the swizzle span); rows past the end read as zero.
bool encode_map(CUtensorMap *m, const void *ptr, CUtensorMapDataType dt, uint64_t esize,
                uint64_t inner, uint64_t rows, uint32_t box_inner) {
  const EncodeTiledFn encode = encode_tiled_fn();
  if (!encode) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * esize};
  cuuint32_t box[2] = {box_inner, (cuuint32_t)C};
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
  const unsigned grid = (unsigned)(p.n_req * p.H);
  auto run = [&](auto kernel) -> cudaError_t {
    const cudaError_t e =
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    kernel<<<grid, NT + 64, SMEM_ALLOC, stream>>>(p, maps);
    return cudaGetLastError();
  };
  const bool logits = p.g_logits != nullptr;
  if (p.local_mode)  // S_loc and M in one pass (no o)
    return logits ? run(prefill_tc_kernel<float, true, true>)
                  : run(prefill_tc_kernel<float, false, true>);
  if (out_dtype == KDA_BF16)
    return logits ? run(prefill_tc_kernel<__nv_bfloat16, true, false>)
                  : run(prefill_tc_kernel<__nv_bfloat16, false, false>);
  return logits ? run(prefill_tc_kernel<float, true, false>)
                : run(prefill_tc_kernel<float, false, false>);
}

}  // namespace kda

#ifdef KDA_PHASE_PROFILE
// Profiling builds only: copy (and optionally clear) the per-phase cycle sums of
// the tensor-core prefill; entry 15 is the number of chunks they cover.
extern "C" int kda_phase_cycles(unsigned long long *out, int n, int clear) {
  if (n > 16) n = 16;
  if (cudaMemcpyFromSymbol(out, kda::g_phase_cycles, n * sizeof(unsigned long long)) !=
      cudaSuccess)
    return 1;
  if (clear) {
    const unsigned long long zero[16] = {};
    if (cudaMemcpyToSymbol(kda::g_phase_cycles, zero, sizeof(zero)) != cudaSuccess) return 1;
  }
  return 0;
}
#endif

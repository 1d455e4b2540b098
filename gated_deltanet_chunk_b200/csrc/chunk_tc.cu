// chunk_tc.cu -- chunked gated-delta-rule forward on the sm_100a tensor cores.
//
// bf16 q/k/v/out, Dk = Dv = 128, chunk C = 64.  One CTA (128 threads) owns one
// (sequence, v-head, 64-column slice of Dv): the recurrence is separable in the
// Dv columns.  The CTA walks its sequence's chunks in order; the fp32 state
// slice S [128 x 64] lives in registers (thread d holds row d) and, rounded to
// bf16, in shared memory as the MMA operand of the next chunk.
//
// Algebra: the chunkwise form of the "手撕Qwen3-Next" walkthrough, section
// 一(一)5(1), steps c-f, with the L2 norms folded into row scales
// (rk = 1/|k|, rq = scale/|q|) so the raw TMA-loaded q/k tiles are the MMA
// operands.  Per chunk (Gamma[r][i] = exp(gcum_r - gcum_i) for i <= r, formed
// only below the diagonal: mask before exp):
//   G  = [Q; K] K^T                                  tcgen05 M=128 N=64  K=128
//   A  = -strictLower(diag(beta rk) (K K^T) diag(rk) * Gamma)          CUDA cores
//   P  = diag(rq) (Q K^T) diag(rk) * Gamma, lower incl. diagonal        CUDA cores
//   T  = (I - A)^-1: with T_D the inverse of A's 16x16 diagonal blocks
//        (forward substitution in registers, warp shuffles) and
//        N = T_D A_off (A_off = the strictly block-lower part),
//        T = (I + N + N^2 + N^3) T_D = R + N^2 R,  R = T_D + N T_D     3 tcgen05 rounds
//        (the 16-row block inverse of the PyPTO README's inverse_pto
//        submodules, with the block merges done as tensor-core products)
//   U  = T diag(beta) V,  W = T diag(beta exp(gcum) rk) K               tcgen05
//   V' = U - W S                                     tcgen05 M=128 N=64  K=128
//   O  = diag(exp(gcum) rq) Q S + P V'               (both accumulate in TMEM)
//   S <- exp(g_last) S + K^T diag(rk exp(g_last - gcum)) V'             tcgen05
// Every accumulation is fp32 in TMEM; MMA operands are bf16.
//
// Operand placement: an M=128 A operand is two stacked 64-row tiles; where only
// 64 rows are meaningful, the other tile is whatever lies next to it in shared
// memory and the matching 64 accumulator rows are ignored.
//
// Every mbarrier wait is bounded (1 s of wall time): on expiry the CTA records
// GDN_ERR_DEVICE_TIMEOUT in a device status word, frees its TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "gdn_common.cuh"
#include "gdn_launch.h"
#include "sm100_ptx.cuh"

namespace gdn {
namespace tc {

__device__ unsigned int g_status;  // bit 0: a bounded wait expired

constexpr int C = 64;
constexpr int DK = 128;
constexpr int DVS = 64;  // Dv columns per CTA
constexpr int kThreads = 128;
constexpr uint64_t kWaitNs = 1000000000ull;

// ---- shared memory layout (bytes from a 1024-aligned base)
constexpr int kTile = 64 * 128;  // 64 rows x 128 bytes (64 bf16)
// one stage: [W_lo | Q_lo | K_lo] [W_hi | Q_hi | K_hi] V P
constexpr int ST_WLO = 0, ST_QLO = 1 * kTile, ST_KLO = 2 * kTile;
constexpr int ST_WHI = 3 * kTile, ST_QHI = 4 * kTile, ST_KHI = 5 * kTile;
constexpr int ST_V = 6 * kTile, ST_P = 7 * kTile;
constexpr int kStage = 8 * kTile;
constexpr int OFF_X0 = 2 * kStage;       // T_D, then R
constexpr int OFF_X1 = OFF_X0 + kTile;   // A_off, then N^2, then T diag(beta)
constexpr int OFF_X2 = OFF_X1 + kTile;   // N, then T diag(beta exp(gcum) rk)
constexpr int OFF_S = OFF_X2 + kTile;    // S operand: 128 rows (d) x 64 cols
constexpr int OFF_VP = OFF_S + 2 * kTile;
constexpr int OFF_WP = OFF_VP + kTile;
constexpr int OFF_SC = OFF_WP + kTile;   // per-row scalars
constexpr int SC_RK = 0, SC_RQ = 64, SC_BETA = 128, SC_GC = 192, SC_EG = 256, SC_WK = 320, SC_BW = 384;
constexpr int OFF_BAR = OFF_SC + 448 * 4;
constexpr int SMEM_USED = OFF_BAR + 64;
constexpr int SMEM_BYTES = SMEM_USED + 1024;  // slack for 1024-byte alignment
static_assert(OFF_BAR % 8 == 0, "mbarrier alignment");
static_assert(SMEM_BYTES <= 232448, "shared memory");

// ---- TMEM columns (128 lanes x 512 fp32 columns)
constexpr uint32_t TM_G = 0, TM_N = 64, TM_N2 = 128, TM_NT = 192, TM_TP = 0;
constexpr uint32_t TM_U = 256, TM_W = 320, TM_D1 = 448, TM_D4 = 64, TM_COLS = 512;

constexpr uint32_t ID_KK64 = ptx::idesc_bf16_f32(128, 64, false, false);
constexpr uint32_t ID_KMN64 = ptx::idesc_bf16_f32(128, 64, false, true);
constexpr uint32_t ID_KMN128 = ptx::idesc_bf16_f32(128, 128, false, true);
constexpr uint32_t ID_MNMN64 = ptx::idesc_bf16_f32(128, 64, true, true);

__device__ __forceinline__ float fast_exp(float x) { return __expf(x); }
__device__ __forceinline__ uint64_t kdesc(uint32_t addr) { return ptx::sdesc_sw128(addr, 16, 1024); }
__device__ __forceinline__ uint64_t mndesc(uint32_t addr, uint32_t lbo) { return ptx::sdesc_sw128(addr, lbo, 1024); }

// K = 64 product: A K-major at a (128 stacked rows), B MN-major at b (K rows of 128 B).
__device__ __forceinline__ void mma_k64(uint32_t d, uint32_t a, uint32_t b, uint32_t b_lbo, uint32_t idesc,
                                        uint32_t acc) {
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) ptx::mma_bf16(d, kdesc(a + 32 * kk), mndesc(b + 2048 * kk, b_lbo), idesc, acc | (kk > 0));
}

__device__ __forceinline__ void tmem_row64(uint32_t taddr, float* v) {
  ptx::tmem_ld32(taddr, v);
  ptx::tmem_ld32(taddr + 32, v + 32);
  ptx::tmem_ld_wait();
}

__global__ void __launch_bounds__(kThreads, 1)
    chunk_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const ChunkArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int slice = blockIdx.x, h = blockIdx.y, n = blockIdx.z;
  const int j = h / (a.nv / a.nqk);
  const int nv = a.nv, dv = a.dv;

  uint64_t* bar_tma = reinterpret_cast<uint64_t*>(sm + OFF_BAR);  // [2]
  uint64_t* bar_mma = bar_tma + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_BAR + 24);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + OFF_BAR + 28);
  float* sc = reinterpret_cast<float*>(sm + OFF_SC);

  int64_t seq_start, seq_end;
  seq_bounds(a.cu, a.uniform_len, n, seq_start, seq_end);
  const int nchunks = (int)((seq_end - seq_start + C - 1) / C);

  if (tid == 0) {
    ptx::mbar_init(bar_tma, 1);
    ptx::mbar_init(bar_tma + 1, 1);
    ptx::mbar_init(bar_mma, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tensormap(&tm_q);
    ptx::prefetch_tensormap(&tm_k);
    ptx::prefetch_tensormap(&tm_v);
  }
  if (warp == 0) {
    ptx::tmem_alloc(tmem_slot, TM_COLS);
    ptx::tmem_relinquish();
  }

  // initial state slice: thread d owns row d (64 fp32)
  float S[64];
  const size_t st_off = ((size_t)n * nv + h) * (size_t)DK * dv + (size_t)tid * dv + slice * DVS;
  if (a.s0) {
    const float4* src = reinterpret_cast<const float4*>(a.s0 + st_off);
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      const float4 x = src[c];
      S[4 * c] = x.x; S[4 * c + 1] = x.y; S[4 * c + 2] = x.z; S[4 * c + 3] = x.w;
    }
  } else {
#pragma unroll
    for (int c = 0; c < 64; ++c) S[c] = 0.f;
  }
  ptx::st_row_bf16(sm + OFF_S, tid, S);
  ptx::fence_proxy_async_smem();
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tl = tmem + ((uint32_t)(32 * warp) << 16);  // this warp's TMEM lane quarter
  const uint32_t sb = ptx::smem_u32(sm);

  auto issue_tma = [&](int chunk, int stage) {
    const int t0 = (int)(seq_start + (int64_t)chunk * C);
    uint8_t* st = sm + stage * kStage;
    uint64_t* bar = bar_tma + stage;
    ptx::mbar_arrive_expect_tx(bar, 5 * kTile);
    ptx::tma_load_3d(st + ST_QLO, &tm_q, bar, 0, j, t0);
    ptx::tma_load_3d(st + ST_QHI, &tm_q, bar, 64, j, t0);
    ptx::tma_load_3d(st + ST_KLO, &tm_k, bar, 0, j, t0);
    ptx::tma_load_3d(st + ST_KHI, &tm_k, bar, 64, j, t0);
    ptx::tma_load_3d(st + ST_V, &tm_v, bar, slice * DVS, h, t0);
  };
  if (tid == 0) {
    if (nchunks > 0) issue_tma(0, 0);
    if (nchunks > 1) issue_tma(1, 1);
  }

  uint32_t mma_phase = 0;
  bool aborted = false;
  // Waits for the last commit; every thread returns the same verdict (after a barrier).
  auto wait_mma = [&]() -> bool {
    if (!ptx::mbar_wait_bounded(bar_mma, mma_phase, kWaitNs)) *abort_flag = 1;
    mma_phase ^= 1u;
    __syncthreads();
    const bool ok = *abort_flag == 0;
    ptx::tc_fence_after();
    return ok;
  };
  auto publish = [&]() {  // thread-written operands -> visible to the tensor cores
    ptx::fence_proxy_async_smem();
    ptx::tc_fence_before();
    __syncthreads();
  };

  // gates of the next chunk (threads 0..63), loaded one chunk ahead
  float g_next = 0.f, b_next = 0.f;
  if (tid < 64 && nchunks > 0) {
    const int64_t t = seq_start + tid;
    if (t < seq_end) {
      g_next = a.g[(size_t)t * nv + h];
      b_next = a.beta[(size_t)t * nv + h];
    }
  }

  for (int ci = 0; ci < nchunks; ++ci) {
    const int stage = ci & 1;
    const int64_t c0 = seq_start + (int64_t)ci * C;
    uint8_t* st = sm + stage * kStage;
    const uint32_t sa = sb + stage * kStage;

    // ---- gates: beta and warp-local cumsum of g (threads 0..63)
    if (tid < 64) {
      float gv = g_next;
      sc[SC_BETA + tid] = b_next;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, gv, o);
        if (lane >= o) gv += y;
      }
      sc[SC_GC + tid] = gv;
      // prefetch the next chunk's gates (latency hidden behind this chunk)
      const int64_t t = c0 + C + tid;
      g_next = 0.f;
      b_next = 0.f;
      if (t < seq_end) {
        g_next = a.g[(size_t)t * nv + h];
        b_next = a.beta[(size_t)t * nv + h];
      }
    }
    if (!ptx::mbar_wait_bounded(bar_tma + stage, (uint32_t)((ci >> 1) & 1), kWaitNs)) *abort_flag = 1;
    __syncthreads();
    if (*abort_flag) { aborted = true; break; }
    // ---- G = [Q; K] K^T
    if (tid == 0) {
      ptx::tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t off = (kk < 4 ? ST_QLO : ST_QHI) + (kk & 3) * 32;
        const uint32_t boff = (kk < 4 ? ST_KLO : ST_KHI) + (kk & 3) * 32;
        ptx::mma_bf16(tmem + TM_G, kdesc(sa + off), kdesc(sa + boff), ID_KK64, kk > 0);
      }
      ptx::mma_commit(bar_mma);
    }
    if (tid >= 32 && tid < 64) sc[SC_GC + tid] += sc[SC_GC + 31];
    // ---- row norms: threads 0..63 queries, 64..127 keys
    {
      const int r = tid & 63;
      const uint8_t* lo = st + (tid < 64 ? ST_QLO : ST_KLO);
      const uint8_t* hi = st + (tid < 64 ? ST_QHI : ST_KHI);
      float v[64];
      float ss = 0.f;
      ptx::ld_row_bf16(lo, r, v);
#pragma unroll
      for (int e = 0; e < 64; ++e) ss = fmaf(v[e], v[e], ss);
      ptx::ld_row_bf16(hi, r, v);
#pragma unroll
      for (int e = 0; e < 64; ++e) ss = fmaf(v[e], v[e], ss);
      const bool valid = c0 + r < seq_end;
      float f = a.qk_l2norm ? 1.f / sqrtf(ss + kNormEps) : 1.f;
      if (tid < 64) f *= a.scale;
      sc[(tid < 64 ? SC_RQ : SC_RK) + r] = valid ? f : 0.f;
    }
    __syncthreads();  // gcum, rk, rq visible
    if (tid < 64) {
      const float gl = sc[SC_GC + 63], gr = sc[SC_GC + tid];
      const float eg = fast_exp(gr);
      sc[SC_EG + tid] = eg;
      sc[SC_WK + tid] = sc[SC_RK + tid] * fast_exp(gl - gr);
      sc[SC_BW + tid] = sc[SC_BETA + tid] * eg * sc[SC_RK + tid];
    }
    if (!wait_mma()) { aborted = true; break; }

    // ---- E1: A rows and the diagonal-block inverse (threads 64..127, key rows);
    //          P rows and Q <- diag(exp(gcum) rq) Q in place (threads 0..63, query rows)
    float td[64];  // key-row threads: row of T_D, later of R
    if (tid >= 64) {
      const int r = tid - 64;
      float av[64];
      tmem_row64(tl + TM_G, av);
      const float fr = -sc[SC_BETA + r] * sc[SC_RK + r];
      const float gr = sc[SC_GC + r];
#pragma unroll
      for (int i = 0; i < 64; ++i) av[i] = (i < r) ? av[i] * fr * sc[SC_RK + i] * fast_exp(gr - sc[SC_GC + i]) : 0.f;
      // diagonal 16x16 block of this row: lanes 0..15 / 16..31 of a warp hold two blocks
      const int li = lane & 15;
      float t[16];
#pragma unroll
      for (int jj = 0; jj < 16; ++jj)
        t[jj] = (warp == 2) ? (lane < 16 ? av[jj] : av[16 + jj]) : (lane < 16 ? av[32 + jj] : av[48 + jj]);
#pragma unroll
      for (int m = 1; m < 15; ++m) {
        const float coef = t[m];
#pragma unroll
        for (int jj = 0; jj < m; ++jj) {
          const float bj = __shfl_sync(0xffffffffu, t[jj], (lane & 16) | m);
          if (li > m) t[jj] = fmaf(coef, bj, t[jj]);
        }
      }
      const int bl = r >> 4;  // block of this row
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const int cb = c >> 4, cj = c & 15;
        td[c] = (cb == bl) ? (cj < li ? t[cj] : (cj == li ? 1.f : 0.f)) : 0.f;
      }
      ptx::st_row_bf16(sm + OFF_X0, r, td);
#pragma unroll
      for (int c = 0; c < 64; ++c) av[c] = (c < 16 * bl) ? av[c] : 0.f;
      ptx::st_row_bf16(sm + OFF_X1, r, av);
    } else {
      const int r = tid;
      float pv[64];
      tmem_row64(tl + TM_G, pv);
      const float fr = sc[SC_RQ + r];
      const float gr = sc[SC_GC + r];
#pragma unroll
      for (int i = 0; i < 64; ++i) pv[i] = (i <= r) ? pv[i] * fr * sc[SC_RK + i] * fast_exp(gr - sc[SC_GC + i]) : 0.f;
      ptx::st_row_bf16(st + ST_P, r, pv);
      const float qf = sc[SC_EG + r] * fr;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint8_t* qt = st + (half ? ST_QHI : ST_QLO);
        ptx::ld_row_bf16(qt, r, pv);
#pragma unroll
        for (int e = 0; e < 64; ++e) pv[e] *= qf;
        ptx::st_row_bf16(qt, r, pv);
      }
    }
    publish();
    // ---- N = T_D A_off   (A operand = [junk; T_D]: rows land in lanes 64..127)
    if (tid == 0) {
      ptx::tc_fence_after();
      mma_k64(tmem + TM_N, sb + OFF_X0 - kTile, sb + OFF_X1, 8192, ID_KMN64, 0);
      ptx::mma_commit(bar_mma);
    }
    if (!wait_mma()) { aborted = true; break; }
    if (tid >= 64) {
      float nv_[64];
      tmem_row64(tl + TM_N, nv_);
      ptx::st_row_bf16(sm + OFF_X2, tid - 64, nv_);
    }
    publish();
    // ---- N^2 = N N,  N T_D
    if (tid == 0) {
      ptx::tc_fence_after();
      mma_k64(tmem + TM_N2, sb + OFF_X2 - kTile, sb + OFF_X2, 8192, ID_KMN64, 0);
      mma_k64(tmem + TM_NT, sb + OFF_X2 - kTile, sb + OFF_X0, 8192, ID_KMN64, 0);
      ptx::mma_commit(bar_mma);
    }
    if (!wait_mma()) { aborted = true; break; }
    if (tid >= 64) {
      float x[64];
      tmem_row64(tl + TM_N2, x);
      ptx::st_row_bf16(sm + OFF_X1, tid - 64, x);
      tmem_row64(tl + TM_NT, x);
#pragma unroll
      for (int c = 0; c < 64; ++c) td[c] += x[c];  // R = T_D + N T_D
      ptx::st_row_bf16(sm + OFF_X0, tid - 64, td);
    }
    publish();
    // ---- T = R + N^2 R
    if (tid == 0) {
      ptx::tc_fence_after();
      mma_k64(tmem + TM_TP, sb + OFF_X1 - kTile, sb + OFF_X0, 8192, ID_KMN64, 0);
      ptx::mma_commit(bar_mma);
    }
    if (!wait_mma()) { aborted = true; break; }
    if (tid >= 64) {
      float x[64];
      tmem_row64(tl + TM_TP, x);
#pragma unroll
      for (int c = 0; c < 64; ++c) x[c] += td[c];
#pragma unroll
      for (int c = 0; c < 64; ++c) td[c] = x[c] * sc[SC_BETA + c];
      ptx::st_row_bf16(sm + OFF_X1, tid - 64, td);  // T diag(beta)
#pragma unroll
      for (int c = 0; c < 64; ++c) td[c] = x[c] * sc[SC_BW + c];
      ptx::st_row_bf16(sm + OFF_X2, tid - 64, td);  // T diag(beta exp(gcum) rk)
    }
    publish();
    // ---- U = T diag(beta) V (rows 0..63) and W = T diag(beta exp(gcum) rk) K (rows 64..127)
    if (tid == 0) {
      ptx::tc_fence_after();
      mma_k64(tmem + TM_U, sb + OFF_X1, sa + ST_V, 8192, ID_KMN64, 0);
      mma_k64(tmem + TM_W, sb + OFF_X1, sa + ST_KLO, ST_KHI - ST_KLO, ID_KMN128, 0);
      ptx::mma_commit(bar_mma);
    }
    if (!wait_mma()) { aborted = true; break; }
    if (tid >= 64) {
      float x[64];
      tmem_row64(tl + TM_W, x);
      ptx::st_row_bf16(st + ST_WLO, tid - 64, x);
      tmem_row64(tl + TM_W + 64, x);
      ptx::st_row_bf16(st + ST_WHI, tid - 64, x);
    }
    publish();
    // ---- D1 = [W; Q'] S : rows 0..63 W S, rows 64..127 diag(exp(gcum) rq) Q S
    if (tid == 0) {
      ptx::tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t off = (kk < 4 ? ST_WLO : ST_WHI) + (kk & 3) * 32;
        ptx::mma_bf16(tmem + TM_D1, kdesc(sa + off), mndesc(sb + OFF_S + 2048 * kk, 8192), ID_KMN64, kk > 0);
      }
      ptx::mma_commit(bar_mma);
    }
    if (!wait_mma()) { aborted = true; break; }
    // ---- V' = U - W S, and diag(rk exp(g_last - gcum)) V' (threads 0..63)
    if (tid < 64) {
      float u[64], ws[64];
      tmem_row64(tl + TM_U, u);
      tmem_row64(tl + TM_D1, ws);
#pragma unroll
      for (int c = 0; c < 64; ++c) u[c] -= ws[c];
      ptx::st_row_bf16(sm + OFF_VP, tid, u);
      const float w = sc[SC_WK + tid];
#pragma unroll
      for (int c = 0; c < 64; ++c) u[c] *= w;
      ptx::st_row_bf16(sm + OFF_WP, tid, u);
    }
    publish();
    // ---- O: D1[64..127] += P V' (A = [V; P]) ;  D4 = K^T W'
    if (tid == 0) {
      ptx::tc_fence_after();
      mma_k64(tmem + TM_D1, sa + ST_V, sb + OFF_VP, 8192, ID_KMN64, 1);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        ptx::mma_bf16(tmem + TM_D4, mndesc(sa + ST_KLO + 2048 * kk, ST_KHI - ST_KLO),
                      mndesc(sb + OFF_WP + 2048 * kk, 8192), ID_MNMN64, kk > 0);
      ptx::mma_commit(bar_mma);
    }
    if (!wait_mma()) { aborted = true; break; }
    // ---- outputs (threads 64..127) and the state update (all threads)
    if (tid >= 64) {
      const int r = tid - 64;
      const int64_t t = c0 + r;
      float o[64];
      tmem_row64(tl + TM_D1, o);
      if (t < seq_end) {
        uint4* orow = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.out) + ((size_t)t * nv + h) * dv +
                                               slice * DVS);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint4 w;
          w.x = ptx::pack_bf16x2(o[8 * c + 0], o[8 * c + 1]);
          w.y = ptx::pack_bf16x2(o[8 * c + 2], o[8 * c + 3]);
          w.z = ptx::pack_bf16x2(o[8 * c + 4], o[8 * c + 5]);
          w.w = ptx::pack_bf16x2(o[8 * c + 6], o[8 * c + 7]);
          orow[c] = w;
        }
      }
    }
    {
      const float decay = fast_exp(sc[SC_GC + 63]);
      float x[64];
      tmem_row64(tl + TM_D4, x);
#pragma unroll
      for (int c = 0; c < 64; ++c) S[c] = fmaf(decay, S[c], x[c]);
      ptx::st_row_bf16(sm + OFF_S, tid, S);
    }
    publish();
    if (tid == 0 && ci + 2 < nchunks) issue_tma(ci + 2, stage);
  }

  if (aborted) {
    if (tid == 0) atomicOr(&g_status, 1u);
  } else if (a.s_final) {
    float4* dst = reinterpret_cast<float4*>(a.s_final + st_off);
#pragma unroll
    for (int c = 0; c < 16; ++c) dst[c] = make_float4(S[4 * c], S[4 * c + 1], S[4 * c + 2], S[4 * c + 3]);
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, TM_COLS);
  }
}

// ---- host side
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 3-D map over a [T, heads, 128] bf16 tensor, box = 64 tokens x 1 head x 64 features.
static bool make_map(CUtensorMap* m, const void* ptr, int heads, int64_t T) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {128, (cuuint64_t)heads, (cuuint64_t)T};
  cuuint64_t strides[2] = {128 * 2, (cuuint64_t)heads * 128 * 2};
  cuuint32_t box[3] = {64, 1, 64};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace tc

bool chunk_tc_supported(int dk, int dv, int chunk, int io_bf16, int64_t total_tokens) {
  return io_bf16 && dk == 128 && dv == 128 && chunk == 64 && total_tokens > 0;
}

cudaError_t launch_chunk_tc(const ChunkArgs& a, int64_t total_tokens, cudaStream_t stream) {
  CUtensorMap mq, mk, mv;
  if (!tc::make_map(&mq, a.q, a.nqk, total_tokens) || !tc::make_map(&mk, a.k, a.nqk, total_tokens) ||
      !tc::make_map(&mv, a.v, a.nv, total_tokens))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(tc::chunk_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       tc::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  dim3 grid(a.dv / tc::DVS, a.nv, a.num_seqs);
  tc::chunk_fwd_tc_kernel<<<grid, tc::kThreads, tc::SMEM_BYTES, stream>>>(mq, mk, mv, a);
  return cudaGetLastError();
}

unsigned int chunk_tc_take_status() {
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, tc::g_status, sizeof(v)) != cudaSuccess) return ~0u;
  if (v) cudaMemcpyToSymbol(tc::g_status, &zero, sizeof(zero));
  return v;
}

}  // namespace gdn

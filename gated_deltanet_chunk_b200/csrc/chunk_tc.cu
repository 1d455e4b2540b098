// chunk_tc.cu -- chunked gated-delta-rule forward on the sm_100a tensor cores.
//
// bf16 q/k/v/out, Dk = Dv = 128, chunk C = 64.  One CTA owns one (sequence,
// v-head, 64-column slice of Dv): the recurrence is separable in the Dv
// columns.  Two warpgroups run a software pipeline over the sequence's chunks:
//
//   intra warpgroup (warps 0-3): everything of chunk c that does not depend on
//     the state -- gate cumsum, L2 norms, G = [K;Q] K^T, the A and P matrices,
//     T = (I - A)^-1, U, W -- runs ahead of the serial warpgroup through a ring
//     of 3 chunk slots in shared memory (plus one TMEM U buffer per slot);
//   serial warpgroup (warps 4-7): the state recurrence, two tensor-core round
//     trips per chunk.  The fp32 state slice S [128 x 64] lives in registers
//     (thread d holds row d) and, rounded to bf16, in shared memory as the B
//     operand of the next chunk.
//
// Algebra: the chunkwise form of the "手撕Qwen3-Next" walkthrough, section
// 一(一)5(1), steps c-f, with the L2 norms folded into row scales
// (rk = 1/|k|, rq = scale/|q|) so the raw TMA-loaded q/k tiles are the MMA
// operands.  Gamma[r][i] = exp(gcum_r - gcum_i) for i <= r is formed only below
// the diagonal (mask before exp), as a product of two factors <= 1 across
// 16-row blocks.  Per chunk:
//   G  = [K; Q] K^T                                     tcgen05 M=128 N=64 K=128
//   A  = -strictLower(diag(beta rk) (K K^T) diag(rk) * Gamma)          CUDA cores
//   P  = diag(rq) (Q K^T) diag(rk) * Gamma, lower incl. diagonal        CUDA cores
//   T  = (I - A)^-1 = R + N^2 R,  R = T_D + N T_D,  N = T_D A_off       3 tcgen05 rounds
//        (T_D: inverse of A's 16x16 diagonal blocks by forward substitution
//        in registers; A_off: the strictly block-lower part of A.  N^4 = 0.
//        The 16-row block scheme is the PyPTO README's inverse_pto submodule.)
//   U  = T diag(beta) V,  W = T diag(beta exp(gcum) rk) K               tcgen05
//   [Q'S ; W S] = [Q'; W] S,  Q' = diag(exp(gcum) rq) Q                  serial
//   V' = U - W S;  O = Q'S + P V'                                        serial
//   S <- exp(g_last) S + K^T diag(rk exp(g_last - gcum)) V'              serial
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
constexpr int DVS = 64;        // Dv columns per CTA
constexpr int kThreads = 256;  // two warpgroups
constexpr int NS = 3;          // chunk slots in flight
constexpr uint64_t kWaitNs = 1000000000ull;

// ---- shared memory layout (bytes from a 1024-aligned base)
constexpr int kTile = 64 * 128;  // 64 rows x 128 bytes (64 bf16)
// one slot: [K_lo | Q_lo | W_lo] [K_hi | Q_hi | W_hi] [V, later P]
constexpr int SL_KLO = 0, SL_QLO = 1 * kTile, SL_WLO = 2 * kTile;
constexpr int SL_KHI = 3 * kTile, SL_QHI = 4 * kTile, SL_WHI = 5 * kTile;
constexpr int SL_VP = 6 * kTile;
constexpr int kSlot = 7 * kTile;
constexpr int OFF_X0 = NS * kSlot;       // intra scratch: A_off, N^2, T diag(bw)
constexpr int OFF_X1 = OFF_X0 + kTile;   // intra scratch: T_D, T diag(beta)
constexpr int OFF_S = OFF_X1 + kTile;    // serial: S operand, 128 rows (d) x 64 cols
constexpr int OFF_VP = OFF_S + 2 * kTile;  // serial: V'
constexpr int OFF_WP = OFF_VP + kTile;     // serial: diag(rk exp(g_last - gcum)) V'
constexpr int OFF_SCI = OFF_WP + kTile;    // intra scalars
constexpr int SI_RK = 0, SI_RQ = 64, SI_BETA = 128, SI_GC = 192, SI_EG = 256, SI_BW = 320, SI_F0 = 384,
              SI_RF = 448, SI_N = 704;  // RF: 4 x 64 table (block 0 unused)
constexpr int OFF_SCS = OFF_SCI + SI_N * 4;  // per-slot scalars for the serial side
constexpr int SS_WK = 0, SS_GAMMA = 64, SS_N = 68;
constexpr int OFF_BAR = OFF_SCS + NS * SS_N * 4;
// barriers: tma_full[NS], slot_free[NS], intra_full[NS], mma_i, mma_s; then tmem slot, abort flag
constexpr int BAR_TMA = 0, BAR_FREE = NS, BAR_INTRA = 2 * NS, BAR_MMAI = 3 * NS, BAR_MMAS = 3 * NS + 1;
constexpr int NBAR = 3 * NS + 2;
constexpr int SMEM_USED = OFF_BAR + NBAR * 8 + 16;
constexpr int SMEM_BYTES = SMEM_USED + 1024;  // slack for 1024-byte alignment
static_assert(OFF_BAR % 8 == 0, "mbarrier alignment");
static_assert(SMEM_BYTES <= 232448, "shared memory");

// ---- TMEM columns (128 lanes x 512 fp32 columns)
constexpr uint32_t TM_G = 0;      // G; then N; then N^2 R
constexpr uint32_t TM_N2 = 64;    // [N^2 | N T_D] (128 cols); then W (128 cols)
constexpr uint32_t TM_U = 192;    // U of slot s at 192 + 64 s
constexpr uint32_t TM_D1 = 384;   // serial: [Q'S ; W S], then O
constexpr uint32_t TM_D4 = 448;   // serial: state update
constexpr uint32_t TM_COLS = 512;

constexpr uint32_t ID_KK64 = ptx::idesc_bf16_f32(128, 64, false, false);
constexpr uint32_t ID_KMN64 = ptx::idesc_bf16_f32(128, 64, false, true);
constexpr uint32_t ID_KMN128 = ptx::idesc_bf16_f32(128, 128, false, true);
constexpr uint32_t ID_MNMN64 = ptx::idesc_bf16_f32(128, 64, true, true);

__device__ __forceinline__ float fast_exp(float x) { return __expf(x); }
__device__ __forceinline__ uint64_t kdesc(uint32_t addr) { return ptx::sdesc_sw128(addr, 16, 1024); }
__device__ __forceinline__ uint64_t mndesc(uint32_t addr, uint32_t lbo) { return ptx::sdesc_sw128(addr, lbo, 1024); }

// K = 64 product: A K-major at a (two stacked 64-row tiles), B MN-major at b.
__device__ __forceinline__ void mma_k64(uint32_t d, uint32_t a, uint32_t b, uint32_t b_lbo, uint32_t idesc,
                                        uint32_t acc) {
#pragma unroll
  for (int kk = 0; kk < 4; ++kk)
    ptx::mma_bf16(d, kdesc(a + 32 * kk), mndesc(b + 2048 * kk, b_lbo), idesc, acc | (kk > 0));
}

__device__ __forceinline__ void tmem_row64(uint32_t taddr, float* v) {
  ptx::tmem_ld32(taddr, v);
  ptx::tmem_ld32(taddr + 32, v + 32);
  ptx::tmem_ld_wait();
}

// row[i] <- row[i] * f * rk_i * Gamma[r][i] for i < r (i <= r when incl_diag), else 0,
// with Gamma[r][i] = exp(gcum_r - gcum_i).  Columns left of r's 16-row block use
// the table RF[b][i] = rk_i exp(gcum_{16b} - gcum_i) times exp(gcum_r - gcum_{16b});
// only the 16 columns of r's own block take a direct exp.  Branch-free: every
// choice is a select on compile-time column indices.
__device__ __forceinline__ void scale_gamma_row(float* row, const float* si, int r, float f, bool incl_diag) {
  const int b = r >> 4, li = r & 15;
  const float gr = si[SI_GC + r];
  const float fb = f * si[SI_F0 + r];
  const float* rf = si + SI_RF + 64 * b;
  const float* gb = si + SI_GC + 16 * b;
  const float* kb = si + SI_RK + 16 * b;
  float own[16];
#pragma unroll
  for (int jj = 0; jj < 16; ++jj) {
    const bool on = incl_diag ? (jj <= li) : (jj < li);
    own[jj] = on ? f * kb[jj] * fast_exp(fminf(gr - gb[jj], 0.f)) : 0.f;
  }
#pragma unroll
  for (int cb = 0; cb < 4; ++cb)
#pragma unroll
    for (int jj = 0; jj < 16; ++jj) {
      const int i = 16 * cb + jj;
      const float fac = (cb < b) ? fb * rf[i] : ((cb == b) ? own[jj] : 0.f);
      row[i] *= fac;
    }
}

__device__ __forceinline__ void named_bar(int id) {
  asm volatile("bar.sync %0, 128;" ::"r"(id) : "memory");
}

__global__ void __launch_bounds__(kThreads, 1)
    chunk_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const ChunkArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // Align within the shared window by pointer arithmetic on the __shared__
  // array, so every access below stays a shared-memory (not generic) access.
  const uint32_t raw_s = ptx::smem_u32(smem_raw);
  uint8_t* sm = smem_raw + (((raw_s + 1023u) & ~1023u) - raw_s);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int slice = blockIdx.x, h = blockIdx.y, n = blockIdx.z;
  const int j = h / (a.nv / a.nqk);
  const int nv = a.nv, dv = a.dv;

  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_BAR + NBAR * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + OFF_BAR + NBAR * 8 + 4);
  float* si = reinterpret_cast<float*>(sm + OFF_SCI);
  float* ss = reinterpret_cast<float*>(sm + OFF_SCS);

  int64_t seq_start, seq_end;
  seq_bounds(a.cu, a.uniform_len, n, seq_start, seq_end);
  const int nchunks = (int)((seq_end - seq_start + C - 1) / C);

  if (tid == 0) {
    for (int i = 0; i < NS; ++i) {
      ptx::mbar_init(bars + BAR_TMA + i, 1);
      ptx::mbar_init(bars + BAR_FREE + i, 1);
      ptx::mbar_init(bars + BAR_INTRA + i, 1);
    }
    ptx::mbar_init(bars + BAR_MMAI, 1);
    ptx::mbar_init(bars + BAR_MMAS, 1);
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
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tl = tmem + ((uint32_t)(32 * (warp & 3)) << 16);  // this warp's TMEM lane quarter
  const uint32_t sb = ptx::smem_u32(sm);

  if (warp < 4) {
    // =====================================================================
    // intra warpgroup
    // =====================================================================
    const int t = tid;  // 0..127
    auto issue_tma = [&](int chunk) {
      const int s = chunk % NS;
      const int t0 = (int)(seq_start + (int64_t)chunk * C);
      uint8_t* sl = sm + s * kSlot;
      uint64_t* bar = bars + BAR_TMA + s;
      ptx::mbar_arrive_expect_tx(bar, 5 * kTile);
      ptx::tma_load_3d(sl + SL_KLO, &tm_k, bar, 0, j, t0);
      ptx::tma_load_3d(sl + SL_KHI, &tm_k, bar, 64, j, t0);
      ptx::tma_load_3d(sl + SL_QLO, &tm_q, bar, 0, j, t0);
      ptx::tma_load_3d(sl + SL_QHI, &tm_q, bar, 64, j, t0);
      ptx::tma_load_3d(sl + SL_VP, &tm_v, bar, slice * DVS, h, t0);
    };
    uint32_t ph_mma = 0;
    bool ok = true;
    // One thread polls the mbarrier; the others park at the named barrier.
    auto wait_bar = [&](uint64_t* bar, uint32_t parity) {
      if (t == 0 && !ptx::mbar_wait_bounded(bar, parity, kWaitNs)) *abort_flag = 1;
      named_bar(1);
      ok = (*abort_flag == 0);
      ptx::tc_fence_after();
    };
    auto wait_mma = [&]() {
      wait_bar(bars + BAR_MMAI, ph_mma);
      ph_mma ^= 1u;
    };
    auto publish = [&]() {
      ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      named_bar(1);
    };

    if (t == 0 && nchunks > 0) issue_tma(0);
    float g_next = 0.f, b_next = 0.f;
    if (t < 64 && seq_start + t < seq_end) {
      g_next = a.g[(size_t)(seq_start + t) * nv + h];
      b_next = a.beta[(size_t)(seq_start + t) * nv + h];
    }

    for (int c = 0; c < nchunks && ok; ++c) {
      const int s = c % NS;
      const int64_t c0 = seq_start + (int64_t)c * C;
      uint8_t* sl = sm + s * kSlot;
      const uint32_t sa = sb + s * kSlot;
      float* sss = ss + s * SS_N;

      // (a) prefetch the next chunk's tiles once its slot is free
      if (t == 0 && c + 1 < nchunks) {
        const int cn = c + 1;
        if (cn >= NS && !ptx::mbar_wait_bounded(bars + BAR_FREE + cn % NS, (uint32_t)((cn / NS - 1) & 1), kWaitNs))
          *abort_flag = 1;
        issue_tma(cn);
      }
      // (b) gates: beta and the warp-local cumsum of g; prefetch the next chunk's gates
      if (t < 64) {
        float gv = g_next;
        si[SI_BETA + t] = b_next;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const float y = __shfl_up_sync(0xffffffffu, gv, o);
          if (lane >= o) gv += y;
        }
        si[SI_GC + t] = gv;
        const int64_t tn = c0 + C + t;
        g_next = 0.f;
        b_next = 0.f;
        if (tn < seq_end) {
          g_next = a.g[(size_t)tn * nv + h];
          b_next = a.beta[(size_t)tn * nv + h];
        }
      }
      // (c) tiles of this chunk
      wait_bar(bars + BAR_TMA + s, (uint32_t)((c / NS) & 1));
      if (!ok) break;
      // (d) G = [K; Q] K^T
      if (t == 0) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t ao = (kk < 4 ? SL_KLO : SL_KHI) + (kk & 3) * 32;
          ptx::mma_bf16(tmem + TM_G, kdesc(sa + ao), kdesc(sa + ao), ID_KK64, kk > 0);
        }
        ptx::mma_commit(bars + BAR_MMAI);
      }
      // (e) norms: threads 0..63 keys (rk), 64..127 queries (rq); cumsum fix-up
      if (t >= 32 && t < 64) si[SI_GC + t] += si[SI_GC + 31];
      {
        const int r = t & 63;
        const uint8_t* lo = sl + (t < 64 ? SL_KLO : SL_QLO);
        const uint8_t* hi = sl + (t < 64 ? SL_KHI : SL_QHI);
        float v[64];
        float sq = 0.f;
        ptx::ld_row_bf16(lo, r, v);
#pragma unroll
        for (int e = 0; e < 64; ++e) sq = fmaf(v[e], v[e], sq);
        ptx::ld_row_bf16(hi, r, v);
#pragma unroll
        for (int e = 0; e < 64; ++e) sq = fmaf(v[e], v[e], sq);
        const bool valid = c0 + r < seq_end;
        float f = a.qk_l2norm ? 1.f / sqrtf(sq + kNormEps) : 1.f;
        if (t >= 64) f *= a.scale;
        si[(t < 64 ? SI_RK : SI_RQ) + r] = valid ? f : 0.f;
      }
      named_bar(1);
      // (f) derived per-row scalars and the cross-block decay table
      if (t < 64) {
        const float gl = si[SI_GC + 63], gr = si[SI_GC + t];
        const float eg = fast_exp(gr);
        const float rk = si[SI_RK + t];
        si[SI_EG + t] = eg;
        si[SI_BW + t] = si[SI_BETA + t] * eg * rk;
        si[SI_F0 + t] = fast_exp(gr - si[SI_GC + (t & ~15)]);  // exp(gcum_r - gcum_{block start})
        sss[SS_WK + t] = rk * fast_exp(gl - gr);
        if (t == 0) sss[SS_GAMMA] = fast_exp(gl);
      } else {
        // RF[b][i] = rk_i exp(gcum_{16b} - gcum_i) for i < 16 b, b = 1..3 (rows of block >= b)
        for (int e = t - 64; e < 256; e += 64) {
          const int b = e >> 6, i = e & 63;
          float val = 0.f;
          if (b >= 1 && i < 16 * b) val = si[SI_RK + i] * fast_exp(si[SI_GC + 16 * b] - si[SI_GC + i]);
          si[SI_RF + e] = val;
        }
      }
      // (g) G ready
      wait_mma();
      if (!ok) break;
      // (h) A rows + diagonal-block inverse (threads 0..63); P rows + Q' in place (threads 64..127)
      // keep[]: query-row threads hold their P row until V has been consumed;
      //         key-row threads hold R = T_D + N T_D for T = R + N^2 R.
      float keep[64];
      float t16[16];   // key-row threads: strictly lower part of this row's T_D block
      if (t < 64) {
        const int r = t, b = r >> 4, li = lane & 15;
        float av[64];
        tmem_row64(tl + TM_G, av);
        const float fr = -si[SI_BETA + r] * si[SI_RK + r];
        scale_gamma_row(av, si, r, fr, false);
#pragma unroll
        for (int jj = 0; jj < 16; ++jj)
          t16[jj] = (warp == 0) ? (lane < 16 ? av[jj] : av[16 + jj]) : (lane < 16 ? av[32 + jj] : av[48 + jj]);
#pragma unroll
        for (int m = 1; m < 15; ++m) {
          const float coef = t16[m];
#pragma unroll
          for (int jj = 0; jj < m; ++jj) {
            const float bj = __shfl_sync(0xffffffffu, t16[jj], (lane & 16) | m);
            if (li > m) t16[jj] = fmaf(coef, bj, t16[jj]);
          }
        }
        float td[64];
#pragma unroll
        for (int cc = 0; cc < 64; ++cc) {
          const int cb = cc >> 4, cj = cc & 15;
          td[cc] = (cb == b) ? (cj < li ? t16[cj] : (cj == li ? 1.f : 0.f)) : 0.f;
        }
        ptx::st_row_bf16(sm + OFF_X1, r, td);
#pragma unroll
        for (int cc = 0; cc < 64; ++cc) av[cc] = (cc < 16 * b) ? av[cc] : 0.f;
        ptx::st_row_bf16(sm + OFF_X0, r, av);
      } else {
        const int r = t - 64, b = r >> 4;
        float* prow = keep;
        tmem_row64(tl + TM_G, prow);
        const float fr = si[SI_RQ + r];
        scale_gamma_row(prow, si, r, fr, true);
        const float qf = si[SI_EG + r] * fr;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint8_t* qt = sl + (half ? SL_QHI : SL_QLO);
          float qv[64];
          ptx::ld_row_bf16(qt, r, qv);
#pragma unroll
          for (int e = 0; e < 64; ++e) qv[e] *= qf;
          ptx::st_row_bf16(qt, r, qv);
        }
      }
      publish();
      // (i) N = T_D A_off   (A = [T_D; junk]: rows land in lanes 0..63)
      if (t == 0) {
        ptx::tc_fence_after();
        mma_k64(tmem + TM_G, sb + OFF_X1, sb + OFF_X0, 8192, ID_KMN64, 0);
        ptx::mma_commit(bars + BAR_MMAI);
      }
      wait_mma();
      if (!ok) break;
      if (t < 64) {
        float x[64];
        tmem_row64(tl + TM_G, x);
        ptx::st_row_bf16(sl + SL_WLO, t, x);  // N (the W slot is free until W is formed)
      }
      publish();
      // (j) [N^2 | N T_D] = N [N | T_D]
      if (t == 0) {
        ptx::tc_fence_after();
        mma_k64(tmem + TM_N2, sa + SL_WLO, sa + SL_WLO, (uint32_t)(OFF_X1 - (s * kSlot + SL_WLO)), ID_KMN128, 0);
        ptx::mma_commit(bars + BAR_MMAI);
      }
      wait_mma();
      if (!ok) break;
      if (t < 64) {
        const int r = t, b = r >> 4, li = lane & 15;
        float x[64];
        tmem_row64(tl + TM_N2, x);
        ptx::st_row_bf16(sm + OFF_X0, r, x);  // N^2
        tmem_row64(tl + TM_N2 + 64, x);
#pragma unroll
        for (int cc = 0; cc < 64; ++cc) {
          const int cb = cc >> 4, cj = cc & 15;
          const float tdv = (cb == b) ? (cj < li ? t16[cj] : (cj == li ? 1.f : 0.f)) : 0.f;
          keep[cc] = tdv + x[cc];  // R = T_D + N T_D
        }
        ptx::st_row_bf16(sl + SL_WHI, r, keep);
      }
      publish();
      // (k) N^2 R
      if (t == 0) {
        ptx::tc_fence_after();
        mma_k64(tmem + TM_G, sb + OFF_X0, sa + SL_WHI, 8192, ID_KMN64, 0);
        ptx::mma_commit(bars + BAR_MMAI);
      }
      wait_mma();
      if (!ok) break;
      if (t < 64) {
        float x[64];
        tmem_row64(tl + TM_G, x);
#pragma unroll
        for (int cc = 0; cc < 64; ++cc) x[cc] += keep[cc];  // T = R + N^2 R
#pragma unroll
        for (int cc = 0; cc < 64; ++cc) keep[cc] = x[cc] * si[SI_BW + cc];
        ptx::st_row_bf16(sm + OFF_X0, t, keep);  // T diag(beta exp(gcum) rk)
#pragma unroll
        for (int cc = 0; cc < 64; ++cc) keep[cc] = x[cc] * si[SI_BETA + cc];
        ptx::st_row_bf16(sm + OFF_X1, t, keep);  // T diag(beta)
      }
      publish();
      // (l) W = T diag(bw) K (rows 0..63), U = T diag(beta) V (rows 64..127 of U[s])
      if (t == 0) {
        ptx::tc_fence_after();
        mma_k64(tmem + TM_U + 64 * s, sb + OFF_X0, sa + SL_VP, 8192, ID_KMN64, 0);
        mma_k64(tmem + TM_N2, sb + OFF_X0, sa + SL_KLO, SL_KHI - SL_KLO, ID_KMN128, 0);
        ptx::mma_commit(bars + BAR_MMAI);
      }
      wait_mma();
      if (!ok) break;
      if (t < 64) {
        float x[64];
        tmem_row64(tl + TM_N2, x);
        ptx::st_row_bf16(sl + SL_WLO, t, x);
        tmem_row64(tl + TM_N2 + 64, x);
        ptx::st_row_bf16(sl + SL_WHI, t, x);
      } else {
        ptx::st_row_bf16(sl + SL_VP, t - 64, keep);  // P row; V has been consumed by U
      }
      publish();
      if (t == 0) ptx::mbar_arrive(bars + BAR_INTRA + s);
    }
    if (!ok && t == 0) atomicOr(&g_status, 1u);
  } else {
    // =====================================================================
    // serial warpgroup
    // =====================================================================
    const int t = tid - 128;  // 0..127: row d of the state
    float S[64];
    const size_t st_off = ((size_t)n * nv + h) * (size_t)DK * dv + (size_t)t * dv + slice * DVS;
    if (a.s0) {
      const float4* src = reinterpret_cast<const float4*>(a.s0 + st_off);
#pragma unroll
      for (int cc = 0; cc < 16; ++cc) {
        const float4 x = src[cc];
        S[4 * cc] = x.x; S[4 * cc + 1] = x.y; S[4 * cc + 2] = x.z; S[4 * cc + 3] = x.w;
      }
    } else {
#pragma unroll
      for (int cc = 0; cc < 64; ++cc) S[cc] = 0.f;
    }
    ptx::st_row_bf16(sm + OFF_S, t, S);
    ptx::fence_proxy_async_smem();
    named_bar(2);

    uint32_t ph_mma = 0;
    bool ok = true;
    auto wait_bar = [&](uint64_t* bar, uint32_t parity) {
      if (t == 0 && !ptx::mbar_wait_bounded(bar, parity, kWaitNs)) *abort_flag = 1;
      named_bar(2);
      ok = (*abort_flag == 0);
      ptx::tc_fence_after();
    };
    auto wait_mma = [&]() {
      wait_bar(bars + BAR_MMAS, ph_mma);
      ph_mma ^= 1u;
    };
    auto publish = [&]() {
      ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      named_bar(2);
    };

    for (int c = 0; c < nchunks && ok; ++c) {
      const int s = c % NS;
      const int64_t c0 = seq_start + (int64_t)c * C;
      const uint32_t sa = sb + s * kSlot;
      const float* sss = ss + s * SS_N;
      wait_bar(bars + BAR_INTRA + s, (uint32_t)((c / NS) & 1));
      if (!ok) break;
      // [Q'; W] S: rows 0..63 Q'S, rows 64..127 W S
      if (t == 0) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t ao = (kk < 4 ? SL_QLO : SL_QHI) + (kk & 3) * 32;
          ptx::mma_bf16(tmem + TM_D1, kdesc(sa + ao), mndesc(sb + OFF_S + 2048 * kk, 8192), ID_KMN64, kk > 0);
        }
        ptx::mma_commit(bars + BAR_MMAS);
      }
      wait_mma();
      if (!ok) break;
      // V' = U - W S and diag(rk exp(g_last - gcum)) V'  (lanes 64..127)
      if (t >= 64) {
        const int r = t - 64;
        float u[64], ws[64];
        tmem_row64(tl + TM_U + 64 * s, u);
        tmem_row64(tl + TM_D1, ws);
#pragma unroll
        for (int cc = 0; cc < 64; ++cc) u[cc] -= ws[cc];
        ptx::st_row_bf16(sm + OFF_VP, r, u);
        const float w = sss[SS_WK + r];
#pragma unroll
        for (int cc = 0; cc < 64; ++cc) u[cc] *= w;
        ptx::st_row_bf16(sm + OFF_WP, r, u);
      }
      publish();
      // O: D1[0..63] += P V' (A = [P; junk]);  D4 = K^T W'
      if (t == 0) {
        ptx::tc_fence_after();
        mma_k64(tmem + TM_D1, sa + SL_VP, sb + OFF_VP, 8192, ID_KMN64, 1);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          ptx::mma_bf16(tmem + TM_D4, mndesc(sa + SL_KLO + 2048 * kk, SL_KHI - SL_KLO),
                        mndesc(sb + OFF_WP + 2048 * kk, 8192), ID_MNMN64, kk > 0);
        ptx::mma_commit(bars + BAR_MMAS);
      }
      wait_mma();
      if (!ok) break;
      // outputs (lanes 0..63) and the state update (all lanes)
      if (t < 64) {
        const int64_t tok = c0 + t;
        float o[64];
        tmem_row64(tl + TM_D1, o);
        if (tok < seq_end) {
          uint4* orow = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.out) + ((size_t)tok * nv + h) * dv +
                                                 slice * DVS);
#pragma unroll
          for (int cc = 0; cc < 8; ++cc) {
            uint4 w;
            w.x = ptx::pack_bf16x2(o[8 * cc + 0], o[8 * cc + 1]);
            w.y = ptx::pack_bf16x2(o[8 * cc + 2], o[8 * cc + 3]);
            w.z = ptx::pack_bf16x2(o[8 * cc + 4], o[8 * cc + 5]);
            w.w = ptx::pack_bf16x2(o[8 * cc + 6], o[8 * cc + 7]);
            orow[cc] = w;
          }
        }
      }
      {
        const float decay = sss[SS_GAMMA];
        float x[64];
        tmem_row64(tl + TM_D4, x);
#pragma unroll
        for (int cc = 0; cc < 64; ++cc) S[cc] = fmaf(decay, S[cc], x[cc]);
        ptx::st_row_bf16(sm + OFF_S, t, S);
      }
      publish();
      if (t == 0) ptx::mbar_arrive(bars + BAR_FREE + s);
    }
    if (ok && a.s_final) {
      float4* dst = reinterpret_cast<float4*>(a.s_final + st_off);
#pragma unroll
      for (int cc = 0; cc < 16; ++cc) dst[cc] = make_float4(S[4 * cc], S[4 * cc + 1], S[4 * cc + 2], S[4 * cc + 3]);
    }
    if (!ok && t == 0) atomicOr(&g_status, 1u);
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

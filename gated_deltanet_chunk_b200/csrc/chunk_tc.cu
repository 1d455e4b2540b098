// chunk_tc.cu -- chunked gated-delta-rule forward on the sm_100a tensor cores.
//
// bf16 q/k/v/out, Dk = Dv = 128, chunk C = 64.  One CTA owns one (sequence,
// v-head, 64-column slice of Dv): the recurrence is separable in the Dv
// columns.  The two CTAs of a (sequence, v-head) form a cluster.  In each CTA:
//
//   intra warps (0-7): the state-independent part of a chunk -- gate cumsum,
//     L2 norms, G = [K;Q] K^T, the A and P matrices and T = (I - A)^-1.
//     Chunk c is built only by cluster rank c % 2, which writes the products
//     (-T diag(bw), P, T diag(beta), per-row scalars) into its own product slot
//     and, with st.async into distributed shared memory, into the same slot of
//     the other CTA, whose mbarrier completes when all those bytes have landed.
//     Each CTA thus builds every other chunk for both Dv slices.
//   serial warps (8-11): the state recurrence for this CTA's Dv slice.  The
//     fp32 state slice S [128 x 64] lives in TMEM (lane d holds row d) and,
//     rounded to bf16, in shared memory as the B operand of the next
//     chunk.  The critical path per chunk is three tensor-core round trips
//     ([K;Q] S, then U and V', then D4) and three short epilogues; W itself
//     is never formed.  P V' is issued by a second thread, so the thread that
//     polls D4 goes straight from issuing it to waiting on it.  The output
//     rows (P V' + Q S) are finished by warps 10-11 while warps 8-9 start the
//     next chunk.  The serial warps also refill this CTA's 3-deep TMA ring of
//     raw q/k/v tiles, and release each product slot (to the other CTA with a
//     relaxed cluster arrive: it reports finished reads, nothing to publish).
//
// Algebra: the chunkwise form of the "手撕Qwen3-Next" walkthrough, section
// 一(一)5(1), steps c-f, with the L2 norms folded into row scales
// (rk = 1/|k|, rq = scale/|q|) so the raw TMA-loaded q/k tiles are the MMA
// operands.  Gamma[r][i] = exp(gcum_r - gcum_i) is formed only for i <= r
// (mask before exp), on the fly while G is scaled.
//   G  = [K; Q] K^T                                     tcgen05 M=128 N=64 K=128
//   A  = -strictLower(diag(beta rk) (K K^T) diag(rk) * Gamma)          CUDA cores
//   P  = diag(rq) (Q K^T) diag(rk) * Gamma  (lower incl. diagonal)      CUDA cores
//   T  = (I - A)^-1: the four 16 x 16 diagonal blocks by forward substitution
//        on T = I + A T in fp32 (one column per lane, one block per warp), then
//        T_10 = T_11 (A_10 T_00) for both 32 x 32 blocks and T21 = T22 (A21 T11)
//        for the whole, as TF32 warp MMAs with fp32 accumulation
//   serial:  [K S; Q S] = [K; Q] S, then U = T diag(beta) V           one round
//            K S rounded to bf16                                      CUDA cores
//            V' = U + (-T diag(beta exp(gcum) rk)) (K S) = U - W S      one round
//            D4 = K^T diag(rk exp(g_last - gcum)) V'                    one round
//            PV = P V'                                            after D4, own use
//            S <- exp(g_last) S + D4;  O = diag(exp(gcum) rq) QS + PV
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

constexpr int C = 64;
constexpr int DK = 128;
constexpr int DVS = 64;        // Dv columns per CTA
constexpr int kThreads = 384;  // 8 intra warps + 4 serial warps
constexpr int NR = 3;          // raw input slots
constexpr int NP = 2;          // product slots
constexpr uint64_t kWaitNs = 1000000000ull;

// ---- shared memory layout (bytes from a 1024-aligned base)
constexpr int kTile = 64 * 128;  // 64 rows x 128 bytes (64 bf16)
// raw slot: [K_lo | Q_lo] [K_hi | Q_hi] V
constexpr int RS_KLO = 0, RS_QLO = 1 * kTile, RS_KHI = 2 * kTile, RS_QHI = 3 * kTile, RS_V = 4 * kTile;
constexpr int kRaw = 5 * kTile;
// product slot: [W_lo | W_hi | P | T diag(beta)].  The builder stores
// -T diag(bw) in W_hi; the serial side forms -W = (-T diag(bw)) K from it into
// W_lo / W_hi, and later overwrites those with V' / W'.
constexpr int PS_WLO = 0, PS_WHI = 1 * kTile, PS_P = 2 * kTile, PS_TU = 3 * kTile;
constexpr int kProd = 4 * kTile;
constexpr int OFF_RAW = 0;
constexpr int OFF_PROD = NR * kRaw;
// intra scratch M: fp32 64 x 64 with rows padded to MS_LD floats, holding A^T,
// then the blocks of T = (I - A)^-1
constexpr int MS_LD = 68;
constexpr int OFF_MS = OFF_PROD + NP * kProd;
constexpr int OFF_S = OFF_MS + 64 * MS_LD * 4;  // serial: S operand, 128 rows (d) x 64 cols
constexpr int OFF_SCI = OFF_S + 2 * kTile;     // intra scalars
constexpr int SI_RK = 0, SI_RQ = 64, SI_BETA = 128, SI_GC = 192, SI_BW = 256, SI_NP = 320, SI_WK = 576,
              SI_SQ = 640, SI_GAM = 704, SI_CF = 708, SI_N = 772;
constexpr int OFF_SCP = OFF_SCI + SI_N * 4;    // per-product-slot scalars for the serial side
constexpr int SP_WK = 0, SP_SQ = 64, SP_GAMMA = 128, SP_N = 132;
// bytes one CTA sends to the other per chunk it builds: -T diag(bw), P, T diag(beta), wk, sq, gamma
constexpr uint32_t kPushBytes = 3 * 8192 + (2 * 64 + 1) * 4;
constexpr int OFF_BAR = OFF_SCP + NP * SP_N * 4;
// barriers: raw_full[NR]; prod_full[NP] (the products of a chunk have landed in
// this CTA); prod_free[NP] (this CTA's serial warps are done with the slot);
// peer_free[NP] (the other CTA's serial warps are done with its copy); mma_i, mma_s
constexpr int BAR_RAWF = 0, BAR_PRODF = NR, BAR_PRODE = NR + NP, BAR_PEERF = NR + 2 * NP;
constexpr int BAR_MMAI = NR + 3 * NP, BAR_MMAS = BAR_MMAI + 1, BAR_MMAD4 = BAR_MMAS + 1, BAR_MMAO = BAR_MMAD4 + 1;
constexpr int BAR_OUTD = BAR_MMAO + 1, BAR_MMAW = BAR_OUTD + 1, BAR_DRAIN = BAR_MMAW + 1, NBAR = BAR_DRAIN + 1;
constexpr int SMEM_USED = OFF_BAR + NBAR * 8 + 16;
constexpr int SMEM_BYTES = SMEM_USED + 1024;  // slack for 1024-byte alignment
static_assert(OFF_BAR % 8 == 0, "mbarrier alignment");
static_assert(SMEM_BYTES <= 232448, "shared memory");

// ---- TMEM columns (128 lanes x 512 fp32 columns)
constexpr uint32_t TM_G = 0;     // intra: G
constexpr uint32_t TM_S = 64;    // serial: the fp32 state slice S (row d in lane d, 64 cols)
constexpr uint32_t TM_QS = 192;  // serial: [K S ; Q S], two column blocks used alternately (128 cols)
constexpr uint32_t TM_U = 320;   // serial: U - W S (rows 0..63)
constexpr uint32_t TM_D4 = 384;  // serial: state update
constexpr uint32_t TM_PV = 448;  // serial: P V' (rows 64..127)
constexpr uint32_t TM_COLS = 512;

constexpr uint32_t ID_KK64 = ptx::idesc_bf16_f32(128, 64, false, false);
constexpr uint32_t ID_KMN64 = ptx::idesc_bf16_f32(128, 64, false, true);
constexpr uint32_t ID_MNMN64 = ptx::idesc_bf16_f32(128, 64, true, true);

// exp(x) as 2^(x log2 e) on the special-function unit, flushing results below
// the fp32 normal range to zero (such decay factors contribute nothing here)
__device__ __forceinline__ float fast_exp(float x) { return ptx::ex2_approx(x * 1.4426950408889634f); }
__device__ __forceinline__ uint64_t kdesc(uint32_t addr) { return ptx::sdesc_sw128(addr, 16, 1024); }
__device__ __forceinline__ uint64_t mndesc(uint32_t addr, uint32_t lbo) { return ptx::sdesc_sw128(addr, lbo, 1024); }

// K = 64 product: A K-major at a (two stacked 64-row tiles), B MN-major at b.
__device__ __forceinline__ void mma_k64(uint32_t d, uint32_t a, uint32_t b, uint32_t b_lbo, uint32_t idesc,
                                        uint32_t acc) {
#pragma unroll
  for (int kk = 0; kk < 4; ++kk)
    ptx::mma_bf16(d, kdesc(a + 32 * kk), mndesc(b + 2048 * kk, b_lbo), idesc, acc | (kk > 0));
}

// K = 128 product: A K-major split in two 64-column tiles at a_lo / a_hi, B MN-major at b.
__device__ __forceinline__ void mma_k128(uint32_t d, uint32_t a_lo, uint32_t a_hi, uint32_t b, uint32_t b_lbo,
                                         uint32_t idesc, uint32_t acc) {
#pragma unroll
  for (int kk = 0; kk < 8; ++kk)
    ptx::mma_bf16(d, kdesc((kk < 4 ? a_lo : a_hi) + 32 * (kk & 3)), mndesc(b + 2048 * kk, b_lbo), idesc,
                  acc | (kk > 0));
}

__device__ __forceinline__ void tmem_row64(uint32_t taddr, float* v) {
  ptx::tmem_ld32(taddr, v);
  ptx::tmem_ld32(taddr + 32, v + 32);
  ptx::tmem_ld_wait();
}

__device__ __forceinline__ void named_bar_n(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Named barrier that also ORs `flag` over the participating threads: every
// participant gets the same answer, so a loop exit decided on it is uniform
// even while another role may be setting the abort flag.
__device__ __forceinline__ bool named_bar_any(int id, int nthreads, bool flag) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)flag), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}


// The sequence this CTA runs: blockIdx.z is a rank, longest sequence first
// (ties by index), so that with packed sequences of mixed lengths, which the
// block scheduler starts in z order, the longest chains start earliest.  Each
// thread ranks one sequence by comparing lengths; beyond kRankMax sequences
// (or with equal lengths) the order is the identity.  Called by all threads.
constexpr int kRankMax = 128;
__device__ __forceinline__ int sequence_of_rank(const ChunkArgs& a, int rank, int* slot) {
  if (a.cu == nullptr || a.num_seqs > kRankMax) return rank;
  if (threadIdx.x == 0) *slot = rank;  // overwritten below; stays only if the ranks were inconsistent
  __syncthreads();
  const int i = threadIdx.x;
  if (i < a.num_seqs) {
    const int li = a.cu[i + 1] - a.cu[i];
    int r = 0;
    for (int q = 0; q < a.num_seqs; ++q) {
      const int lq = a.cu[q + 1] - a.cu[q];
      r += (lq > li) || (lq == li && q < i);
    }
    if (r == rank) *slot = i;
  }
  __syncthreads();
  return *slot;
}

template <bool kRawGate>
__global__ void __launch_bounds__(kThreads, 1)
    chunk_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const ChunkArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // Align within the shared window by pointer arithmetic on the __shared__
  // array, so every access below stays a shared-memory (not generic) access.
  const uint32_t raw_s = ptx::smem_u32(smem_raw);
  uint8_t* sm = smem_raw + (((raw_s + 1023u) & ~1023u) - raw_s);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int slice = blockIdx.x, h = blockIdx.y;
  const int j = h / (a.nv / a.nqk);
  const int nv = a.nv, dv = a.dv;

  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + OFF_BAR + NBAR * 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + OFF_BAR + NBAR * 8 + 4);
  int* seq_slot = reinterpret_cast<int*>(sm + OFF_BAR + NBAR * 8 + 8);
  const int n = sequence_of_rank(a, (int)blockIdx.z, seq_slot);
  float* si = reinterpret_cast<float*>(sm + OFF_SCI);
  float* sp = reinterpret_cast<float*>(sm + OFF_SCP);

  int64_t seq_start, seq_end;
  seq_bounds(a, n, seq_start, seq_end);
  const int nchunks = (int)((seq_end - seq_start + C - 1) / C);

  const uint32_t crank = ptx::cluster_ctarank();  // == slice
  const uint32_t peer = crank ^ 1u;
  if (tid == 0) {
    for (int i = 0; i < NR; ++i) ptx::mbar_init(bars + BAR_RAWF + i, 1);
    for (int i = 0; i < NP; ++i) {
      ptx::mbar_init(bars + BAR_PRODF + i, 1);
      ptx::mbar_init(bars + BAR_PRODE + i, 1);
      ptx::mbar_init(bars + BAR_PEERF + i, 1);
    }
    ptx::mbar_init(bars + BAR_MMAI, 1);
    ptx::mbar_init(bars + BAR_MMAS, 1);
    ptx::mbar_init(bars + BAR_MMAD4, 1);
    ptx::mbar_init(bars + BAR_MMAO, 1);
    ptx::mbar_init(bars + BAR_OUTD, 2);
    ptx::mbar_init(bars + BAR_MMAW, 1);
    ptx::mbar_init(bars + BAR_DRAIN, 3);  // one commit per MMA-issuing thread
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
  ptx::cluster_sync_all();  // both CTAs' barriers are initialised before any remote arrive
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tl = tmem + ((uint32_t)(32 * (warp & 3)) << 16);  // this warp's TMEM lane quarter
  const uint32_t sb = ptx::smem_u32(sm);

  if (warp < 8) {
    // =====================================================================
    // intra warps (0-7): thread (quarter q = warp % 4, half h = warp / 4, lane)
    // owns accumulator row 32q + lane of G, columns [16h, 16h + 16) and
    // [32 + 16h, 48 + 16h).
    // =====================================================================
    const int t = tid;  // 0..255
    const int q = warp & 3, hf = warp >> 2;
    const int row = 32 * q + lane;  // accumulator row: 0..63 keys, 64..127 queries
    const int r = row & 63;
    const bool krow = q < 2;
    float* ms = reinterpret_cast<float*>(sm + OFF_MS);
    uint32_t ph_mma = 0;
    bool ok = true;
    // One thread polls the mbarrier; the others park at the named barrier.
    auto wait_bar = [&](uint64_t* bar, uint32_t parity) {
      if (t == 0 && !ptx::mbar_wait_bounded(bar, parity, kWaitNs)) *abort_flag = 1;
      ok = !named_bar_any(1, 256, *abort_flag != 0);
      ptx::tc_fence_after();
    };
    float g_next = 0.f, b_next = 0.f;
    {
      const int64_t t0g = seq_start + (int64_t)crank * C + t;
      if (t < 64 && t0g < seq_end) {
        load_gate_t<kRawGate>(a, (size_t)t0g * nv + h, h, g_next, b_next);
      }
    }

    // this CTA builds the chunks c with c % 2 == cluster rank
    for (int c = (int)crank; c < nchunks && ok; c += 2) {
      const int rsl = c % NR, psl = c % NP;
      const int64_t c0t = seq_start + (int64_t)c * C;
      uint8_t* rs = sm + OFF_RAW + rsl * kRaw;
      const uint32_t ra = sb + OFF_RAW + rsl * kRaw;
      uint8_t* ps = sm + OFF_PROD + psl * kProd;
      const uint32_t pa = sb + OFF_PROD + psl * kProd;
      float* spp = sp + psl * SP_N;
      const uint32_t rpa = ptx::mapa(pa, peer);                     // the other CTA's copy of the slot
      const uint32_t rspp = ptx::mapa(ptx::smem_u32(spp), peer);
      const uint32_t rbar = ptx::mapa(ptx::smem_u32(bars + BAR_PRODF + psl), peer);  // the other CTA's prod_full

      // gates: beta and the warp-local cumsum of g; prefetch the next chunk's gates
      if (t < 64) {
        float gv = g_next;
        // checked here, a chunk after the load was issued, so the check does not wait for it
        if (!(gv <= 0.f)) report_status(a.status, kStatusGate);  // the decay factoring needs g <= 0
        si[SI_BETA + t] = b_next;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const float y = __shfl_up_sync(0xffffffffu, gv, o);
          if (lane >= o) gv += y;
        }
        si[SI_GC + t] = gv;
        const int64_t tn = c0t + 2 * C + t;  // this CTA's next chunk
        g_next = 0.f;
        b_next = 0.f;
        if (tn < seq_end) {
          load_gate_t<kRawGate>(a, (size_t)tn * nv + h, h, g_next, b_next);
        }
      }
      wait_bar(bars + BAR_RAWF + rsl, (uint32_t)((c / NR) & 1));
      if (!ok) break;
      // G = [K; Q] K^T
      if (t == 0) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t ao = (kk < 4 ? RS_KLO : RS_KHI) + (kk & 3) * 32;
          ptx::mma_bf16(tmem + TM_G, kdesc(ra + ao), kdesc(ra + ao), ID_KK64, kk > 0);
        }
        ptx::mma_commit(bars + BAR_MMAI);
      }
      if (t >= 32 && t < 64) si[SI_GC + t] += si[SI_GC + 31];
      // norms: half-row partial sums (threads 0..127 low halves, 128..255 high halves)
      {
        const int nr = t & 127, part = t >> 7;
        const uint8_t* tile = rs + (nr < 64 ? (part ? RS_KHI : RS_KLO) : (part ? RS_QHI : RS_QLO));
        float v[64];
        float sq = 0.f;
        ptx::ld_row_bf16(tile, nr & 63, v);
#pragma unroll
        for (int e = 0; e < 64; ++e) sq = fmaf(v[e], v[e], sq);
        si[SI_NP + t] = sq;
      }
      named_bar_n(1, 256);
      if (t < 128) {
        const int nr = t & 63;
        const float sq = si[SI_NP + t] + si[SI_NP + 128 + t];
        const bool valid = c0t + nr < seq_end;
        float f = a.qk_l2norm ? 1.f / sqrtf(sq + kNormEps) : 1.f;
        if (t >= 64) f *= a.scale;
        si[(t < 64 ? SI_RK : SI_RQ) + nr] = valid ? f : 0.f;
      }
      named_bar_n(1, 256);
      // row scalars; CF_i = rk_i exp(gcum_b - gcum_i) with b = the last column
      // of i's 32-column half (the pivot for rows below that half)
      if (t < 64) {
        const float gl = si[SI_GC + 63], gr = si[SI_GC + t];
        const float eg = fast_exp(gr);
        const float rk = si[SI_RK + t];
        si[SI_CF + t] = rk * fast_exp(si[SI_GC + (t | 31)] - gr);
        si[SI_BW + t] = si[SI_BETA + t] * eg * rk;
        si[SI_WK + t] = rk * fast_exp(gl - gr);
        si[SI_SQ + t] = eg * si[SI_RQ + t];
        if (t == 0) si[SI_GAM] = fast_exp(gl);
      }
      wait_bar(bars + BAR_MMAI, ph_mma);  // G ready (the barrier also publishes the scalars)
      ph_mma ^= 1u;
      if (!ok) break;
      // A rows (key rows) go to the fp32 scratch M for the inverse; P rows
      // (query rows) wait in registers, packed to bf16, until the slot is free
      uint4 pk0[4];
      {
        // G row r, scaled to A (key rows) or P (query rows):
        //   A[r][i] = -beta_r rk_r rk_i exp(gcum_r - gcum_i) (K K^T)[r][i],  i < r
        //   P[r][i] =  rq_r rk_i exp(gcum_r - gcum_i) (Q K^T)[r][i],        i <= r
        // The thread takes 16 columns from each 32-column block, [16 hf, 16 hf + 16)
        // and [32 + 16 hf, 48 + 16 hf), so every warp has one 16-column run in its
        // rows' diagonal block.  The decay is formed only where i <= r (mask before
        // exp); for a run in the block left of the diagonal block (rows 32..63,
        // columns < 32) it is split at column 31, exp(gcum_r - gcum_31)
        // exp(gcum_31 - gcum_i), both factors <= 1 for gates <= 0.
        float av[32];
        ptx::tmem_ld16(tl + TM_G + 16 * hf, av);
        ptx::tmem_ld16(tl + TM_G + 32 + 16 * hf, av + 16);
        ptx::tmem_ld_wait();
        ptx::tc_fence_before();  // G is consumed: the next chunk's G may overwrite it after any barrier
        const float f = krow ? -si[SI_BETA + r] * si[SI_RK + r] : si[SI_RQ + r];
        const int rblk = r >> 5;  // == q & 1: warp-uniform
        // the run in the diagonal block, columns [cd, cd + 16) (both branches below
        // index av with constants, keeping it in registers)
        auto diag_run = [&](float* dg, int cd) {
          const float gr = si[SI_GC + r];
          const int lim = krow ? r : r + 1;  // columns i < lim are kept
          const float4* rk4 = reinterpret_cast<const float4*>(si + SI_RK + cd);
          const float4* gc4 = reinterpret_cast<const float4*>(si + SI_GC + cd);
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {
            const float4 rk = rk4[k4], gc = gc4[k4];
            const int i0 = cd + 4 * k4;
            dg[4 * k4 + 0] = (i0 + 0 < lim) ? dg[4 * k4 + 0] * (f * rk.x) * fast_exp(gr - gc.x) : 0.f;
            dg[4 * k4 + 1] = (i0 + 1 < lim) ? dg[4 * k4 + 1] * (f * rk.y) * fast_exp(gr - gc.y) : 0.f;
            dg[4 * k4 + 2] = (i0 + 2 < lim) ? dg[4 * k4 + 2] * (f * rk.z) * fast_exp(gr - gc.z) : 0.f;
            dg[4 * k4 + 3] = (i0 + 3 < lim) ? dg[4 * k4 + 3] * (f * rk.w) * fast_exp(gr - gc.w) : 0.f;
          }
        };
        if (rblk == 1) {
          const float rowf = f * fast_exp(si[SI_GC + r] - si[SI_GC + 31]);
          const float4* cf = reinterpret_cast<const float4*>(si + SI_CF + 16 * hf);
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {
            const float4 x = cf[k4];
            av[4 * k4 + 0] *= rowf * x.x;
            av[4 * k4 + 1] *= rowf * x.y;
            av[4 * k4 + 2] *= rowf * x.z;
            av[4 * k4 + 3] *= rowf * x.w;
          }
          diag_run(av + 16, 32 + 16 * hf);
        } else {
          diag_run(av, 16 * hf);
#pragma unroll
          for (int cc = 16; cc < 32; ++cc) av[cc] = 0.f;  // above the diagonal block
        }
        if (krow) {
          // M[i][r] = A[r][i] (column i of A is row i of M); the 32 x 32 block above
          // the diagonal is zero and never read
          float* mc = ms + 16 * hf * MS_LD + r;
#pragma unroll
          for (int cc = 0; cc < 16; ++cc) mc[cc * MS_LD] = av[cc];
          if (rblk == 1) {
#pragma unroll
            for (int cc = 0; cc < 16; ++cc) mc[(32 + cc) * MS_LD] = av[16 + cc];
          }
        } else {
          ptx::pack_half_bf16(av, pk0);  // P: chunks 2 hf, 2 hf + 1, 4 + 2 hf, 5 + 2 hf of the row
        }
      }
      // the product slot (both copies) must have been released by both CTAs'
      // serial warps (chunk c - 2) before this chunk's products are stored
      if (t == 0) {
        if (c >= NP) {
          const uint32_t par = (uint32_t)((c / NP - 1) & 1);
          if (!ptx::mbar_wait_bounded(bars + BAR_PRODE + psl, par, kWaitNs)) *abort_flag = 1;
          if (!ptx::mbar_wait_cluster_bounded(bars + BAR_PEERF + psl, par, kWaitNs)) *abort_flag = 1;
        }
      }
      ok = !named_bar_any(1, 256, *abort_flag != 0);  // also: A^T is in M
      if (!ok) break;
      // arm the other CTA's copy, off the inverse's path (bytes that land first
      // only drive the count below zero; the phase cannot complete before this
      // arrival, and the previous phase completed before the slot was released)
      if (t == 64) ptx::mbar_arrive_expect_tx_remote(rbar, kPushBytes);
      // T = (I - A)^-1 by blocks (A is strictly lower triangular, T unit lower
      // triangular).  M holds A^T on entry; each T block is written over an A^T
      // block that is no longer needed, ending with T11, T22 row-major in M's
      // diagonal 32 x 32 blocks (their upper right 16 x 16 still holds A^T and is
      // read as zero) and T21 in block (0, 1).
      //   1. the four 16 x 16 diagonal blocks in fp32 on the CUDA cores, T = I + A T
      //      from the top, one per warp (0, 1, 4, 5; one column per lane);
      //      meanwhile warps 2, 3, 6, 7 store P, whose rows they hold
      //   2. both 32 x 32 diagonal blocks: T_10 = T_11 (A_10 T_00) on 16 x 16 blocks
      //   3. T21 = T22 (A21 T11) on 32 x 32 blocks
      // Steps 2 and 3 are TF32 warp MMAs with fp32 accumulation (T is rounded to
      // bf16 as an MMA operand afterwards, far coarser than TF32's 2^-11).
      if (krow) {
        const int b = (warp & 1) | ((warp >> 2) << 1);  // warps 0, 1, 4, 5 -> blocks 0..3
        float* mb = ms + 16 * b * MS_LD + 16 * b;       // row k of this block of M = column k of A_bb
        if (lane < 16) {
          float x[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) x[i] = (i == lane) ? 1.f : 0.f;
          float4 cur[4], nxt[4];
#pragma unroll
          for (int v = 0; v < 4; ++v) cur[v] = *reinterpret_cast<const float4*>(mb + 4 * v);
#pragma unroll
          for (int k = 0; k < 15; ++k) {
            if (k + 1 < 15) {
#pragma unroll
              for (int v = (k + 2) >> 2; v < 4; ++v)
                nxt[v] = *reinterpret_cast<const float4*>(mb + (k + 1) * MS_LD + 4 * v);
            }
#pragma unroll
            for (int i = k + 1; i < 16; ++i) {
              const float4 y = cur[i >> 2];
              const float aik = (i & 3) == 0 ? y.x : (i & 3) == 1 ? y.y : (i & 3) == 2 ? y.z : y.w;
              x[i] = fmaf(aik, x[k], x[i]);
            }
#pragma unroll
            for (int v = 0; v < 4; ++v) cur[v] = nxt[v];
          }
          __syncwarp(0x0000ffffu);
#pragma unroll
          for (int i = 0; i < 16; ++i) mb[i * MS_LD + lane] = x[i];  // T_bb, row-major
        }
      } else {
#pragma unroll
        for (int c = 0; c < 4; ++c)  // P
          *reinterpret_cast<uint4*>(ps + PS_P + ptx::sw128_off(r, 2 * hf + (c & 1) + 4 * (c >> 1))) = pk0[c];
        ptx::fence_proxy_async_smem();
#pragma unroll
        for (int c = 0; c < 4; ++c)
          ptx::st_async_v4(rpa + PS_P + ptx::sw128_off(r, 2 * hf + (c & 1) + 4 * (c >> 1)), pk0[c], rbar);
      }
      named_bar_n(1, 256);
      // 2. both 32 x 32 diagonal blocks: T_10 = T_11 (A_10 T_00) on 16 x 16 blocks,
      //    warps 0-3 = (pair, 8-column tile), TF32 warp MMAs; Y = A_10 T_00 is
      //    kept where A^T is zero (rows 16..31, columns 0..15 of the pair's block)
      //    and then overwritten by T_10
      const int g8 = lane >> 2, t4 = lane & 3;
      if (warp < 4) {
        const int pp = warp >> 1, nt = warp & 1;
        float* base = ms + 32 * pp * MS_LD + 32 * pp;
        float y[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k0 = 0; k0 < 16; k0 += 8) {
          uint32_t af[4], bf[2];
          af[0] = ptx::to_tf32(base[(k0 + t4) * MS_LD + 16 + g8]);      // A_10[g][k] = M[k][16 + g]
          af[1] = ptx::to_tf32(base[(k0 + t4) * MS_LD + 24 + g8]);
          af[2] = ptx::to_tf32(base[(k0 + t4 + 4) * MS_LD + 16 + g8]);
          af[3] = ptx::to_tf32(base[(k0 + t4 + 4) * MS_LD + 24 + g8]);
          bf[0] = ptx::to_tf32(base[(k0 + t4) * MS_LD + 8 * nt + g8]);  // T_00[k][n]
          bf[1] = ptx::to_tf32(base[(k0 + t4 + 4) * MS_LD + 8 * nt + g8]);
          ptx::mma_tf32_16x8x8(y, af, bf);
        }
        float* yo = base + 16 * MS_LD + 8 * nt + 2 * t4;
        yo[g8 * MS_LD] = y[0];
        yo[g8 * MS_LD + 1] = y[1];
        yo[(g8 + 8) * MS_LD] = y[2];
        yo[(g8 + 8) * MS_LD + 1] = y[3];
        __syncwarp();
        float z[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k0 = 0; k0 < 16; k0 += 8) {
          uint32_t af[4], bf[2];
          af[0] = ptx::to_tf32(base[(16 + g8) * MS_LD + 16 + k0 + t4]);  // T_11[g][k]
          af[1] = ptx::to_tf32(base[(24 + g8) * MS_LD + 16 + k0 + t4]);
          af[2] = ptx::to_tf32(base[(16 + g8) * MS_LD + 20 + k0 + t4]);
          af[3] = ptx::to_tf32(base[(24 + g8) * MS_LD + 20 + k0 + t4]);
          bf[0] = ptx::to_tf32(base[(16 + k0 + t4) * MS_LD + 8 * nt + g8]);  // Y[k][n]
          bf[1] = ptx::to_tf32(base[(20 + k0 + t4) * MS_LD + 8 * nt + g8]);
          ptx::mma_tf32_16x8x8(z, af, bf);
        }
        __syncwarp();  // every lane has read Y
        yo[g8 * MS_LD] = z[0];
        yo[g8 * MS_LD + 1] = z[1];
        yo[(g8 + 8) * MS_LD] = z[2];
        yo[(g8 + 8) * MS_LD + 1] = z[3];
      }
      named_bar_n(1, 256);
      // 3. T21 = T22 (A21 T11) on 32 x 32 blocks: warp -> (16-row tile mt, 8-column
      //    tile nt); T11 and T22 hold A^T values above their diagonal 16 x 16
      //    blocks, so their upper triangles are masked to T's zeros as they are read
      {
        const int mt = warp >> 2, nt = warp & 3;
        const int ra0 = 16 * mt + g8, cb = 8 * nt + g8;
        float y[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k0 = 0; k0 < 32; k0 += 8) {
          uint32_t af[4], bf[2];
          af[0] = ptx::to_tf32(ms[(k0 + t4) * MS_LD + 32 + ra0]);  // A21[i][k] = M[k][32 + i]
          af[1] = ptx::to_tf32(ms[(k0 + t4) * MS_LD + 40 + ra0]);
          af[2] = ptx::to_tf32(ms[(k0 + t4 + 4) * MS_LD + 32 + ra0]);
          af[3] = ptx::to_tf32(ms[(k0 + t4 + 4) * MS_LD + 40 + ra0]);
          const int kb0 = k0 + t4, kb1 = k0 + t4 + 4;
          bf[0] = ptx::to_tf32(cb <= kb0 ? ms[kb0 * MS_LD + cb] : 0.f);  // T11[k][n], lower triangle
          bf[1] = ptx::to_tf32(cb <= kb1 ? ms[kb1 * MS_LD + cb] : 0.f);
          ptx::mma_tf32_16x8x8(y, af, bf);
        }
        float* yo = ms + (32 + ra0) * MS_LD + 8 * nt + 2 * t4;  // Y over A^T's zero block
        yo[0] = y[0];
        yo[1] = y[1];
        yo[8 * MS_LD] = y[2];
        yo[8 * MS_LD + 1] = y[3];
        named_bar_n(1, 256);
        float z[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k0 = 0; k0 < 32; k0 += 8) {
          uint32_t af[4], bf[2];
          const int ka = k0 + t4, kb = k0 + t4 + 4;
          af[0] = ptx::to_tf32(ka <= ra0 ? ms[(32 + ra0) * MS_LD + 32 + ka] : 0.f);  // T22[i][k], lower
          af[1] = ptx::to_tf32(ka <= ra0 + 8 ? ms[(40 + ra0) * MS_LD + 32 + ka] : 0.f);
          af[2] = ptx::to_tf32(kb <= ra0 ? ms[(32 + ra0) * MS_LD + 32 + kb] : 0.f);
          af[3] = ptx::to_tf32(kb <= ra0 + 8 ? ms[(40 + ra0) * MS_LD + 32 + kb] : 0.f);
          bf[0] = ptx::to_tf32(ms[(32 + ka) * MS_LD + cb]);  // Y[k][n]
          bf[1] = ptx::to_tf32(ms[(32 + kb) * MS_LD + cb]);
          ptx::mma_tf32_16x8x8(z, af, bf);
        }
        float* zo = ms + ra0 * MS_LD + 32 + 8 * nt + 2 * t4;  // T21 into block (0, 1)
        zo[0] = z[0];
        zo[1] = z[1];
        zo[8 * MS_LD] = z[2];
        zo[8 * MS_LD + 1] = z[3];
      }
      named_bar_n(1, 256);  // T21 is in M
      // products: stored locally first (and made visible to this CTA's tensor
      // cores), then sent to the other CTA with st.async
      if (t < 64) {
        spp[SP_WK + t] = si[SI_WK + t];
        spp[SP_SQ + t] = si[SI_SQ + t];
        if (t == 0) spp[SP_GAMMA] = si[SI_GAM];
      }
      {
        // every thread a quarter row of T (row pr, columns [16 qc, 16 qc + 16));
        // P was stored while the diagonal blocks were solved
        const int pr = t & 63, qc = t >> 6, ph = qc >> 1, sub = qc & 1;
        float x[16];
        if (pr < 32 && ph == 1) {
#pragma unroll
          for (int cc = 0; cc < 16; ++cc) x[cc] = 0.f;
        } else {
          const float* tr =
              ms + (pr < 32 ? pr * MS_LD : (ph == 0 ? (pr - 32) * MS_LD + 32 : pr * MS_LD + 32)) + 16 * sub;
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const float4 y = *reinterpret_cast<const float4*>(tr + 4 * v);
            x[4 * v] = y.x; x[4 * v + 1] = y.y; x[4 * v + 2] = y.z; x[4 * v + 3] = y.w;
          }
          if ((pr >> 5) == ph) {  // a diagonal 32 x 32 block: T is zero above the diagonal
            const int lim = (pr & 31) - 16 * sub;
#pragma unroll
            for (int cc = 0; cc < 16; ++cc) x[cc] = cc <= lim ? x[cc] : 0.f;
          }
        }
        float y[16];
        uint4 wv[2], tu[2];
#pragma unroll
        for (int cc = 0; cc < 16; ++cc) y[cc] = -x[cc] * si[SI_BW + 16 * qc + cc];
        wv[0] = ptx::pack8_bf16(y);  // -T diag(beta exp(gcum) rk), for W
        wv[1] = ptx::pack8_bf16(y + 8);
#pragma unroll
        for (int cc = 0; cc < 16; ++cc) y[cc] = x[cc] * si[SI_BETA + 16 * qc + cc];
        tu[0] = ptx::pack8_bf16(y);  // T diag(beta), for U
        tu[1] = ptx::pack8_bf16(y + 8);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          *reinterpret_cast<uint4*>(ps + PS_WHI + ptx::sw128_off(pr, 2 * qc + c)) = wv[c];
          *reinterpret_cast<uint4*>(ps + PS_TU + ptx::sw128_off(pr, 2 * qc + c)) = tu[c];
        }
        ptx::fence_proxy_async_smem();
        if (t < 64) {
          ptx::st_async_b32(rspp + 4 * (SP_WK + t), __float_as_uint(si[SI_WK + t]), rbar);
          ptx::st_async_b32(rspp + 4 * (SP_SQ + t), __float_as_uint(si[SI_SQ + t]), rbar);
          if (t == 0) ptx::st_async_b32(rspp + 4 * SP_GAMMA, __float_as_uint(si[SI_GAM]), rbar);
        }
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          ptx::st_async_v4(rpa + PS_WHI + ptx::sw128_off(pr, 2 * qc + c), wv[c], rbar);
          ptx::st_async_v4(rpa + PS_TU + ptx::sw128_off(pr, 2 * qc + c), tu[c], rbar);
        }
      }
      named_bar_n(1, 256);
      if (t == 0) ptx::mbar_arrive(bars + BAR_PRODF + psl);  // the other CTA's copy completes by transactions
    }
    if (!ok && t == 0) report_status(a.status, kStatusTimeout);
  } else {
    // =====================================================================
    // serial warps (8-11)
    // =====================================================================
    const int t = tid - 256;  // 0..127: row d of the state
    // S lives in TMEM (fp32) and, rounded to bf16, in shared memory
    const int64_t srow = state_row(a, n);  // -1: a padding sequence (zero state, nothing stored)
    const size_t st_off = ((size_t)(srow < 0 ? 0 : srow) * nv + h) * (size_t)DK * dv + (size_t)t * dv + slice * DVS;
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      float x[32];
      if (a.s0 && srow >= 0) {
        const float4* src = reinterpret_cast<const float4*>(a.s0 + st_off + 32 * hh);
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) {
          const float4 y = src[cc];
          x[4 * cc] = y.x; x[4 * cc + 1] = y.y; x[4 * cc + 2] = y.z; x[4 * cc + 3] = y.w;
        }
      } else {
#pragma unroll
        for (int cc = 0; cc < 32; ++cc) x[cc] = 0.f;
      }
      ptx::tmem_st32(tl + TM_S + 32 * hh, x);
      ptx::st_half_bf16(sm + OFF_S, t, hh, x);
    }
    ptx::tmem_st_wait();
    ptx::fence_proxy_async_smem();
    named_bar_n(2, 128);

    bool ok = true;
    // this CTA's raw q/k/v tiles of chunk `chunk` (slot chunk % NR)
    auto issue_tma = [&](int chunk) {
      const int s = chunk % NR;
      const int t0 = (int)(seq_start + (int64_t)chunk * C);
      uint8_t* rs = sm + OFF_RAW + s * kRaw;
      uint64_t* bar = bars + BAR_RAWF + s;
      ptx::mbar_arrive_expect_tx(bar, 5 * kTile);
      ptx::tma_load_3d(rs + RS_KLO, &tm_k, bar, 0, j, t0);
      ptx::tma_load_3d(rs + RS_KHI, &tm_k, bar, 64, j, t0);
      ptx::tma_load_3d(rs + RS_QLO, &tm_q, bar, 0, j, t0);
      ptx::tma_load_3d(rs + RS_QHI, &tm_q, bar, 64, j, t0);
      ptx::tma_load_3d(rs + RS_V, &tm_v, bar, slice * DVS, h, t0);
    };
    int issued = 0;    // chunks whose tiles have been requested (thread 64)
    int consumed = 0;  // chunks whose tiles are known to have landed
    if (t == 64)
      for (; issued < NR && issued < nchunks; ++issued) issue_tma(issued);
    // warps 8-9 own the token rows of U - W S (TMEM lanes 0..63); warps 10-11
    // the output rows (lanes 64..127).  Per chunk every thread passes the same
    // barriers whether or not a wait has expired, and all four warps leave the
    // loop together at the second 128-thread barrier.
    const bool vrow = t < 64;

    for (int c = 0; c < nchunks; ++c) {
      const int rsl = c % NR, psl = c % NP;
      const uint32_t par = (uint32_t)(c & 1);
      const uint32_t ra = sb + OFF_RAW + rsl * kRaw;
      uint8_t* ps = sm + OFF_PROD + psl * kProd;
      const uint32_t pa = sb + OFF_PROD + psl * kProd;
      const float* spp = sp + psl * SP_N;
      const uint32_t tm_qs = TM_QS + 64u * par;  // [K S; Q S] alternates between two column blocks
      if (vrow) {
        // [K S; Q S], committed alone so that the K S epilogue need not wait
        // for U = T diag(beta) V, issued after it (the tensor pipe runs one
        // thread's MMAs in order; the commit of the next round covers U)
        if (t == 0) {
          if (!ptx::mbar_wait_bounded(bars + BAR_RAWF + rsl, (uint32_t)((c / NR) & 1), kWaitNs) ||
              !ptx::mbar_wait_cluster_bounded(bars + BAR_PRODF + psl, (uint32_t)((c / NP) & 1), kWaitNs))
            *abort_flag = 1;
          if (*abort_flag == 0) {
            ptx::fence_proxy_async_smem();  // products stored by threads (possibly of the other CTA)
            ptx::tc_fence_after();
            mma_k128(tmem + tm_qs, ra + RS_KLO, ra + RS_KHI, sb + OFF_S, 8192, ID_KMN64, 0);
            ptx::mma_commit(bars + BAR_MMAW);
            mma_k64(tmem + TM_U, pa + PS_TU, ra + RS_V, 8192, ID_KMN64, 0);
            if (!ptx::mbar_wait_bounded(bars + BAR_MMAW, par, kWaitNs)) *abort_flag = 1;
          }
        }
        named_bar_n(3, 64);
        ok = (*abort_flag == 0);
        ptx::tc_fence_after();
        if (ok) {
          // row t of K S, rounded to bf16, into W_lo: the B operand of the next product
          float x[64];
          tmem_row64(tl + tm_qs, x);
          ptx::st_row_bf16(ps + PS_WLO, t, x);
        }
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        named_bar_n(3, 64);
        // V' = U + (-T diag(bw)) (K S) = U - W S   (A = [-T diag(bw); junk])
        if (t == 0) {
          if (*abort_flag == 0) {
            ptx::tc_fence_after();
            mma_k64(tmem + TM_U, pa + PS_WHI, pa + PS_WLO, 8192, ID_KMN64, 1);
            ptx::mma_commit(bars + BAR_MMAS);
            if (!ptx::mbar_wait_bounded(bars + BAR_MMAS, par, kWaitNs)) *abort_flag = 1;
          }
        }
        named_bar_n(3, 64);
        ok = (*abort_flag == 0);
        ptx::tc_fence_after();
        if (ok) {
          // V' = U - W S and W' = diag(rk exp(g_last - gcum)) V'  (into the W tiles)
          const float w = spp[SP_WK + t];
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            float u[32];
            ptx::tmem_ld32(tl + TM_U + 32 * hh, u);
            ptx::tmem_ld_wait();
            ptx::st_half_bf16(ps + PS_WLO, t, hh, u);
#pragma unroll
            for (int cc = 0; cc < 32; ++cc) u[cc] *= w;
            ptx::st_half_bf16(ps + PS_WHI, t, hh, u);
          }
        }
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        named_bar_n(3, 64);
        if (t == 0 && *abort_flag == 0) {
          // D4 = K^T W' (the recurrence), then P V' (A = [junk; P]: rows land in
          // lanes 64..127) once the output warps have read the previous one
          ptx::tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            ptx::mma_bf16(tmem + TM_D4, mndesc(ra + RS_KLO + 2048 * kk, RS_KHI - RS_KLO),
                          mndesc(pa + PS_WHI + 2048 * kk, 8192), ID_MNMN64, kk > 0);
          ptx::mma_commit(bars + BAR_MMAD4);
        }
        if (t == 32 && *abort_flag == 0) {  // off the polling thread's path
          ptx::tc_fence_after();
          if (c > 0 && !ptx::mbar_wait_bounded(bars + BAR_OUTD, par ^ 1u, kWaitNs)) *abort_flag = 1;
          ptx::tc_fence_after();
          mma_k64(tmem + TM_PV, pa + PS_P - kTile, pa + PS_WLO, 8192, ID_KMN64, 0);
          ptx::mma_commit(bars + BAR_MMAO);
        }
      }
      // S <- exp(g_last) S + D4   (thread t owns row t)
      if (t == 0 && *abort_flag == 0 && !ptx::mbar_wait_bounded(bars + BAR_MMAD4, par, kWaitNs)) *abort_flag = 1;
      named_bar_n(2, 128);
      ok = (*abort_flag == 0);
      ptx::tc_fence_after();
      if (ok) {
        consumed = c + 1;
        const float decay = spp[SP_GAMMA];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          float x[32], sv[32];
          ptx::tmem_ld32(tl + TM_D4 + 32 * hh, x);
          ptx::tmem_ld32(tl + TM_S + 32 * hh, sv);
          ptx::tmem_ld_wait();
#pragma unroll
          for (int cc = 0; cc < 32; ++cc) sv[cc] = fmaf(decay, sv[cc], x[cc]);
          ptx::tmem_st32(tl + TM_S + 32 * hh, sv);
          ptx::st_half_bf16(sm + OFF_S, t, hh, sv);
        }
        ptx::tmem_st_wait();
      }
      ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      ok = !named_bar_any(2, 128, *abort_flag != 0);
      if (!ok) break;
      if (!vrow) {
        // output rows, off the recurrence's critical path:
        // O = diag(exp(gcum) rq) Q S + P V'
        const int orow = t - 64;
        const int64_t tok = seq_start + (int64_t)c * C + orow;
        if (t == 64) {
          if (c + NR < nchunks) {  // every read of this raw slot has completed (D4 was the last)
            issue_tma(c + NR);
            issued = c + NR + 1;
          }
          if (!ptx::mbar_wait_bounded(bars + BAR_MMAO, par, kWaitNs)) *abort_flag = 1;
        }
        const float f = spp[SP_SQ + orow];  // read before the slot is released below
        named_bar_n(4, 64);
        const bool ook = (*abort_flag == 0);
        ptx::tc_fence_after();
        if (t == 64) {
          // release the product slot to the CTA that builds chunk c + 2
          if ((c & 1) == (int)crank)
            ptx::mbar_arrive(bars + BAR_PRODE + psl);
          else
            ptx::mbar_arrive_remote_relaxed(ptx::mapa(ptx::smem_u32(bars + BAR_PEERF + psl), peer));
        }
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
          float qs[16], pv[16];
          if (ook) {
            ptx::tmem_ld16(tl + tm_qs + 16 * qq, qs);
            ptx::tmem_ld16(tl + TM_PV + 16 * qq, pv);
            ptx::tmem_ld_wait();
          }
          if (qq == 3) {  // both accumulators have been read: they may be overwritten
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bars + BAR_OUTD);
          }
          if (ook && tok < seq_end) {
            uint4* op = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.out) + ((size_t)tok * nv + h) * dv +
                                                 slice * DVS + 16 * qq);
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
              uint4 w;
              w.x = ptx::pack_bf16x2(fmaf(f, qs[8 * cc + 0], pv[8 * cc + 0]), fmaf(f, qs[8 * cc + 1], pv[8 * cc + 1]));
              w.y = ptx::pack_bf16x2(fmaf(f, qs[8 * cc + 2], pv[8 * cc + 2]), fmaf(f, qs[8 * cc + 3], pv[8 * cc + 3]));
              w.z = ptx::pack_bf16x2(fmaf(f, qs[8 * cc + 4], pv[8 * cc + 4]), fmaf(f, qs[8 * cc + 5], pv[8 * cc + 5]));
              w.w = ptx::pack_bf16x2(fmaf(f, qs[8 * cc + 6], pv[8 * cc + 6]), fmaf(f, qs[8 * cc + 7], pv[8 * cc + 7]));
              op[cc] = w;
            }
          }
        }
      }
    }
    if (!ok && t == 64) {
      // abort: let the tile loads still in flight land before this CTA exits (bounded)
      for (int cn = consumed; cn < issued; ++cn)
        ptx::mbar_wait_bounded(bars + BAR_RAWF + cn % NR, (uint32_t)((cn / NR) & 1), kWaitNs);
    }
    if (ok && a.s_final && srow >= 0) {
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        float x[32];
        ptx::tmem_ld32(tl + TM_S + 32 * hh, x);
        ptx::tmem_ld_wait();
        float4* dst = reinterpret_cast<float4*>(a.s_final + st_off + 32 * hh);
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) dst[cc] = make_float4(x[4 * cc], x[4 * cc + 1], x[4 * cc + 2], x[4 * cc + 3]);
      }
    }
    if (!ok && t == 0) report_status(a.status, kStatusTimeout);
  }

  // Every thread that issued MMAs (intra 0, serial 0 and 32) commits once more:
  // on an early exit some of its MMAs may still be running, and TMEM is freed
  // only after they have completed (bounded, like every wait here).
  if (tid == 0 || tid == 256 || tid == 288) ptx::mma_commit(bars + BAR_DRAIN);
  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync_all();  // the other CTA no longer touches this CTA's shared memory
  if (warp == 0) {
    if (lane == 0 && !ptx::mbar_wait_bounded(bars + BAR_DRAIN, 0u, kWaitNs)) report_status(a.status, kStatusTimeout);
    __syncwarp();
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

bool chunk_tc_supported(int dk, int dv, int chunk, int io_bf16) {
  return io_bf16 && dk == 128 && dv == 128 && chunk == 64;
}

cudaError_t launch_chunk_tc(const ChunkArgs& a, int64_t total_tokens, cudaStream_t stream) {
  CUtensorMap mq, mk, mv;
  if (!tc::make_map(&mq, a.q, a.nqk, total_tokens) || !tc::make_map(&mk, a.k, a.nqk, total_tokens) ||
      !tc::make_map(&mv, a.v, a.nv, total_tokens))
    return cudaErrorInvalidValue;
  const bool raw_gate = a.A_log != nullptr;
  auto kernel = raw_gate ? tc::chunk_fwd_tc_kernel<true> : tc::chunk_fwd_tc_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, tc::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.dv / tc::DVS, a.nv, a.num_seqs);  // x: the two Dv slices = one cluster
  cfg.blockDim = dim3(tc::kThreads, 1, 1);
  cfg.dynamicSmemBytes = tc::SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kernel, mq, mk, mv, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// Self-test of the failure detection: one CTA waits, with the same bounded
// mbarrier wait the chunk kernel uses, on a barrier nothing arrives on; after
// limit_ns it gives up and records the timeout in the status word.
__global__ void selftest_wait_kernel(uint64_t limit_ns, unsigned int* status) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    ptx::mbar_init(&bar, 1);
    ptx::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !ptx::mbar_wait_bounded(&bar, 0u, limit_ns)) report_status(status, kStatusTimeout);
}

cudaError_t launch_selftest_wait(uint64_t limit_ns, unsigned int* status, cudaStream_t s) {
  selftest_wait_kernel<<<1, 32, 0, s>>>(limit_ns, status);
  return cudaGetLastError();
}

}  // namespace gdn

// chunk_simt.cu -- chunked gated-delta-rule forward with fp32 CUDA-core arithmetic.
//
// This is the kernel for the fp32 io path (and any shape the tensor-core kernel
// does not take).  It follows the chunkwise algorithm of the "手撕Qwen3-Next"
// walkthrough, section 一(一)5(1) (torch_chunk_gated_delta_rule), with two
// re-associations that avoid materialising W and the output attention's
// separate U term:
//
//   V' = U - W S = T diag(beta) (V - diag(exp(gcum)) K S)          (step e/f)
//   o  = diag(exp(gcum)) Q S + P V',  P = (Q K^T * Gamma), lower incl. diagonal
//   S <- exp(g_last) S + (K * exp(g_last - gcum))^T V'
//
// where T = (I - A)^-1 (the walkthrough's step d, which forms it by a row
// recursion; here by 16 x 16 diagonal blocks and doubling merges),
// A = -strictLower(diag(beta) (K K^T * Gamma)), Gamma = exp(gcum_r - gcum_i)
// for i <= r (mask before exp), gcum = in-chunk inclusive cumsum of g (step c).
//
// One CTA owns one (sequence, v-head, 32-column slice of Dv): the state
// recurrence is separable in the Dv columns, so slices are independent.  The
// CTA walks its sequence's chunks in order, keeping the fp32 state slice
// [Dk x 32] in shared memory.  Rows past the sequence end behave as
// q = k = v = g = beta = 0 (the walkthrough's zero padding), which leaves the
// state unchanged.
#include "gdn_common.cuh"
#include "gdn_launch.h"
#include "sm100_ptx.cuh"

namespace gdn {
namespace simt {

constexpr int kThreads = 256;
constexpr int kDVS = 32;  // Dv columns per CTA

template <int C, int DK>
struct Smem {
  static constexpr int AP = C + 1;                // padded pitch of A / T / P rows
  static constexpr int kKhT = 0;                  // [DK][C] keys, transposed, swizzled
  static constexpr int kQhT = kKhT + DK * C;      // [DK][C] queries, transposed, swizzled
  static constexpr int kA = kQhT + DK * C;        // [C][AP] A, then T - I, then P
  static constexpr int kS = kA + C * AP;          // [DK][kDVS] state slice
  static constexpr int kV = kS + DK * kDVS;       // [C][kDVS] X, then V'
  static constexpr int kGc = kV + C * kDVS;       // [C] gcum
  static constexpr int kBeta = kGc + C;           // [C] beta
  static constexpr int kEg = kBeta + C;           // [C] exp(gcum)
  static constexpr int kEkl = kEg + C;            // [C] exp(g_last - gcum)
  static constexpr int kTotal = kEkl + C;
  static constexpr size_t kBytes = size_t(kTotal) * sizeof(float);
  static_assert(kS % 4 == 0 && kV % 4 == 0, "float4 alignment");
  static_assert(kBytes <= 232448, "shared memory budget");
};

// Transposed [D][C] tile with a 16-byte XOR swizzle: element (d, r).
template <int C>
__device__ __forceinline__ int swz(int d, int r) {
  return d * C + ((((r >> 2) ^ (d & 7))) << 2) + (r & 3);
}

template <int C>
__device__ __forceinline__ float4 ld4_t(const float* base, int d, int r0) {
  return *reinterpret_cast<const float4*>(base + swz<C>(d, r0));
}

// fp32 x = hi + lo with hi, lo both TF32 (the low 13 bits of each are zero):
// products of such splits, hi hi + hi lo + lo hi, are within about 2^-22 of
// the exact product, so three TF32 MMAs stand in for fp32 ones.  That is four
// times fp32's rounding: the key-key and query-key dot products (A and P
// below), whose cancellation sets the relative accuracy of short or nearly
// orthogonal sequences' outputs, stay on fp32 FMAs.
__device__ __forceinline__ void split_tf32(float x, uint32_t& hi, uint32_t& lo) {
  hi = ptx::to_tf32(x);
  lo = ptx::to_tf32(x - __uint_as_float(hi));
}

// acc[NT] (16 x 8 fp32 tiles, columns 8 j .. 8 j + 7 of a 16 x 8 NT block) +=
// A[16 x K] B[K x 8 NT] over k in [k0, k1) (multiples of 8), one warp, with
// a(m, k) and b(k, n) reading the operands' elements (m < 16, n < 8 NT).
template <int NT, typename FA, typename FB>
__device__ __forceinline__ void warp_mma_3xtf32(float (&acc)[NT][4], int k0, int k1, FA a, FB b, int g, int t) {
#pragma unroll 2
  for (int kk = k0; kk < k1; kk += 8) {
    uint32_t ah[4], al[4];
    split_tf32(a(g, kk + t), ah[0], al[0]);
    split_tf32(a(g + 8, kk + t), ah[1], al[1]);
    split_tf32(a(g, kk + t + 4), ah[2], al[2]);
    split_tf32(a(g + 8, kk + t + 4), ah[3], al[3]);
#pragma unroll
    for (int jj = 0; jj < NT; ++jj) {
      uint32_t bh[2], bl[2];
      split_tf32(b(kk + t, 8 * jj + g), bh[0], bl[0]);
      split_tf32(b(kk + t + 4, 8 * jj + g), bh[1], bl[1]);
      ptx::mma_tf32_16x8x8(acc[jj], al, bh);
      ptx::mma_tf32_16x8x8(acc[jj], ah, bl);
      ptx::mma_tf32_16x8x8(acc[jj], ah, bh);
    }
  }
}

// A (IS_P = false):  A[r][i] = -beta_r (k_r . k_i) Gamma[r][i] for i < r, else 0.
// P (IS_P = true):   P[r][i] = (q_r . k_i) Gamma[r][i] for i <= r, else 0.
template <int C, int DK, bool IS_P>
__device__ __forceinline__ void pair_matrix(float* sm, int tid) {
  using L = Smem<C, DK>;
  const float* X = sm + (IS_P ? L::kQhT : L::kKhT);
  const float* Kt = sm + L::kKhT;
  const float* gc = sm + L::kGc;
  const float* bt = sm + L::kBeta;
  float* A = sm + L::kA;
  // Only the 4 x 4 tiles on or below the diagonal are formed (numbered row by
  // row: tile tl is (rt, it) with tl = rt (rt + 1) / 2 + it, it <= rt).  The
  // warp MMAs that read A (as T - I) and P take whole 16 x 16 diagonal blocks,
  // so the entries above the diagonal tiles inside those blocks are zeroed;
  // nothing reads further up.
  for (int e = tid; e < (C / 16) * 256; e += kThreads) {
    const int b = e >> 8, r = (e >> 4) & 15, i = e & 15;
    if ((i >> 2) > (r >> 2)) A[(16 * b + r) * L::AP + 16 * b + i] = 0.f;
  }
  constexpr int NTC = C / 4, NL = NTC * (NTC + 1) / 2;
  for (int tl = tid; tl < NL; tl += kThreads) {
    int rt = (int)((sqrtf(8.f * (float)tl + 1.f) - 1.f) * 0.5f);
    while ((rt + 1) * (rt + 2) / 2 <= tl) ++rt;
    while (rt * (rt + 1) / 2 > tl) --rt;
    const int r0 = rt * 4, i0 = (tl - rt * (rt + 1) / 2) * 4;
    float acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) acc[a][b] = 0.f;
    {
#pragma unroll 4
      for (int d = 0; d < DK; ++d) {
        const float4 x = ld4_t<C>(X, d, r0);
        const float4 y = ld4_t<C>(Kt, d, i0);
        const float xs[4] = {x.x, x.y, x.z, x.w};
        const float ys[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
          for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(xs[a], ys[b], acc[a][b]);
      }
    }
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int r = r0 + a, i = i0 + b;
        float val = 0.f;
        if (IS_P ? (i <= r) : (i < r)) {
          val = acc[a][b] * expf(gc[r] - gc[i]);  // masked before exp: gc[r] - gc[i] <= 0
          if (!IS_P) val = -bt[r] * val;
        }
        A[r * L::AP + i] = val;
      }
  }
}

// T - I for T = (I - A)^-1, A strictly lower triangular (held in A, pitch AP),
// written over A.  The walkthrough's row recursion (section 一(一)5(1) d) has
// C - 1 dependent steps; here the same T comes from its block form:
//   1. each 16 x 16 diagonal block by forward substitution, one warp per block
//      and one column per lane: (T - I)[i][j] = A[i][j] + sum_{j<m<i} A[i][m] (T - I)[m][j];
//   2. doubling the solved blocks, for s = 16, 32, ... < C: a diagonal block
//      [[T00, 0], [T10, T11]] of size 2s has T10 = T11 A10 T00, formed as
//      Y = A10 + A10 (T00 - I), then T10 = Y + (T11 - I) Y (warp MMAs below).
// Y needs s x s floats per pair (C s / 2 in all), held in the V tile, which
// is free until X is formed.
template <int C, int DK>
__device__ __forceinline__ void invert_blocked(float* sm, int tid) {
  using L = Smem<C, DK>;
  constexpr int AP = L::AP;
  float* A = sm + L::kA;
  float* Y = sm + L::kV;
  static_assert(C / 16 <= kThreads / 32, "one warp per diagonal block");
  static_assert(C * C / 4 <= C * kDVS, "Y fits in the V tile");
  const int lane = tid & 31, warp = tid >> 5;
  if (warp < C / 16 && lane < 16) {
    float* blk = A + (16 * warp) * AP + 16 * warp;
    const int jc = lane;
    float x[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      float acc = (jc < i) ? blk[i * AP + jc] : 0.f;
#pragma unroll
      for (int m = 0; m < i; ++m)
        if (m > jc) acc = fmaf(blk[i * AP + m], x[m], acc);
      x[i] = acc;
    }
    __syncwarp(0x0000ffffu);
#pragma unroll
    for (int i = 0; i < 16; ++i)
      if (jc < i) blk[i * AP + jc] = x[i];
  }
  __syncthreads();
  // the doubling merges as warp MMAs (TF32 split three ways): a unit is one
  // pair's 16 x 16 output block (two 16 x 8 tiles); phase 1 forms Y, phase 2 T10
#pragma unroll 1
  for (int s = 16; s < C; s *= 2) {
    const int nb = s / 16, nunit = (C / (2 * s)) * nb * nb;
    const int g = lane >> 2, t = lane & 3;
    for (int u = warp; u < nunit; u += kThreads / 32) {
      const int p = u / (nb * nb), rb = (u / nb) % nb, cb = u % nb;
      const int base = 2 * s * p;
      const float* a10 = A + (base + s + 16 * rb) * AP + base;  // rows 16 rb.. of A10
      const float* t00 = A + base * AP + base + 16 * cb;         // (T00 - I), columns 16 cb..
      float acc[2][4] = {};
      // (T00 - I)[k][j] is zero for k <= j: k starts at the column block
      warp_mma_3xtf32<2>(acc, 16 * cb, s, [&](int m, int kk) { return a10[m * AP + kk]; },
                         [&](int kk, int n) { return t00[kk * AP + n]; }, g, t);
      float* yp = Y + p * s * s;
#pragma unroll
      for (int jj = 0; jj < 2; ++jj)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int m = 16 * rb + g + 8 * (e >> 1), jc = 16 * cb + 8 * jj + 2 * t + (e & 1);
          yp[m * s + jc] = a10[(g + 8 * (e >> 1)) * AP + jc] + acc[jj][e];
        }
    }
    __syncthreads();
    for (int u = warp; u < nunit; u += kThreads / 32) {
      const int p = u / (nb * nb), rb = (u / nb) % nb, cb = u % nb;
      const int base = 2 * s * p;
      const float* t11 = A + (base + s + 16 * rb) * AP + base + s;  // rows 16 rb.. of (T11 - I)
      const float* yp = Y + p * s * s;
      float acc[2][4] = {};
      // (T11 - I)[i][m] is zero for m >= i: columns up to the row block's end
      warp_mma_3xtf32<2>(acc, 0, 16 * rb + 16, [&](int m, int kk) { return t11[m * AP + kk]; },
                         [&](int kk, int n) { return yp[kk * s + 16 * cb + n]; }, g, t);
      float* t10 = A + (base + s) * AP + base;
#pragma unroll
      for (int jj = 0; jj < 2; ++jj)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int m = 16 * rb + g + 8 * (e >> 1), jc = 16 * cb + 8 * jj + 2 * t + (e & 1);
          t10[m * AP + jc] = yp[m * s + jc] + acc[jj][e];
        }
    }
    __syncthreads();
  }
}

template <int C, int DK, typename IO>
__global__ void __launch_bounds__(kThreads, 1) chunk_fwd_simt_kernel(ChunkArgs a) {
  using L = Smem<C, DK>;
  extern __shared__ __align__(16) float sm[];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cslice = blockIdx.x * kDVS;  // first Dv column of this CTA
  const int h = blockIdx.y;              // v-head
  const int n = blockIdx.z;              // sequence
  const int j = h / (a.nv / a.nqk);      // qk-head
  const IO* q = static_cast<const IO*>(a.q);
  const IO* k = static_cast<const IO*>(a.k);
  const IO* v = static_cast<const IO*>(a.v);
  IO* out = static_cast<IO*>(a.out);
  const int dv = a.dv;
  const int nv = a.nv, nqk = a.nqk;

  int64_t seq_start, seq_end;
  seq_bounds(a, n, seq_start, seq_end);

  float* S = sm + L::kS;
  float* KhT = sm + L::kKhT;
  float* QhT = sm + L::kQhT;
  float* A = sm + L::kA;
  float* V = sm + L::kV;
  float* gc = sm + L::kGc;
  float* bt = sm + L::kBeta;
  float* eg = sm + L::kEg;
  float* ekl = sm + L::kEkl;

  const int64_t srow = state_row(a, n);  // -1: a padding sequence (zero state, nothing stored)
  const size_t state_off = ((size_t)(srow < 0 ? 0 : srow) * nv + h) * (size_t)DK * dv;
  for (int e = tid; e < DK * kDVS; e += kThreads) {
    const int d = e / kDVS, c = e % kDVS;
    S[e] = (a.s0 && srow >= 0) ? a.s0[state_off + (size_t)d * dv + cslice + c] : 0.f;
  }

  for (int64_t c0 = seq_start; c0 < seq_end; c0 += C) {
    __syncthreads();  // previous chunk fully consumed
    // ---- load q, k rows; L2 norm (eps inside the root) and query scale ----
    // RB rows per warp at a time, so that their loads are in flight together
    constexpr int PER = DK / 32, RB = 4;
    static_assert(C % ((kThreads / 32) * RB) == 0, "rows per pass");
    for (int r0 = warp * RB; r0 < C; r0 += (kThreads / 32) * RB) {
      float qv[RB][PER], kv[RB][PER], sq[RB], sk[RB];
#pragma unroll
      for (int rb = 0; rb < RB; ++rb) {
        const int64_t t = c0 + r0 + rb;
        const bool valid = t < seq_end;
        // lane l holds elements l, l + 32, ...: each load is one coalesced row
        // segment, and the transposed stores below spread over the banks
        const size_t off = ((size_t)(valid ? t : 0) * nqk + j) * DK + lane;
#pragma unroll
        for (int e = 0; e < PER; ++e) {
          qv[rb][e] = valid ? to_f32(q[off + 32 * e]) : 0.f;
          kv[rb][e] = valid ? to_f32(k[off + 32 * e]) : 0.f;
        }
      }
#pragma unroll
      for (int rb = 0; rb < RB; ++rb) {
        sq[rb] = 0.f;
        sk[rb] = 0.f;
#pragma unroll
        for (int e = 0; e < PER; ++e) {
          sq[rb] = fmaf(qv[rb][e], qv[rb][e], sq[rb]);
          sk[rb] = fmaf(kv[rb][e], kv[rb][e], sk[rb]);
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int rb = 0; rb < RB; ++rb) {
          sq[rb] += __shfl_xor_sync(0xffffffffu, sq[rb], o);
          sk[rb] += __shfl_xor_sync(0xffffffffu, sk[rb], o);
        }
#pragma unroll
      for (int rb = 0; rb < RB; ++rb) {
        const int r = r0 + rb;
        const float fq = (a.qk_l2norm ? 1.f / sqrtf(sq[rb] + kNormEps) : 1.f) * a.scale;
        const float fk = a.qk_l2norm ? 1.f / sqrtf(sk[rb] + kNormEps) : 1.f;
#pragma unroll
        for (int e = 0; e < PER; ++e) {
          const int d = 32 * e + lane;
          QhT[swz<C>(d, r)] = qv[rb][e] * fq;
          KhT[swz<C>(d, r)] = kv[rb][e] * fk;
        }
      }
    }
    if (tid < C) {
      const int64_t t = c0 + tid;
      const bool valid = t < seq_end;
      float gv = 0.f, bv = 0.f;
      if (valid) load_gate(a, (size_t)t * nv + h, h, gv, bv);
      gc[tid] = gv;
      bt[tid] = bv;
    }
    __syncthreads();
    // ---- in-chunk inclusive cumsum of g (one warp) ----
    if (warp == 0) {
      constexpr int PG = C / 32;
      float loc[PG];
      float run = 0.f;
#pragma unroll
      for (int e = 0; e < PG; ++e) {
        run += gc[lane * PG + e];
        loc[e] = run;
      }
      float incl = run;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      float excl = __shfl_up_sync(0xffffffffu, incl, 1);
      if (lane == 0) excl = 0.f;
#pragma unroll
      for (int e = 0; e < PG; ++e) gc[lane * PG + e] = loc[e] + excl;
    }
    __syncthreads();
    if (tid < C) {
      const float glast = gc[C - 1];
      eg[tid] = expf(gc[tid]);
      ekl[tid] = expf(glast - gc[tid]);
    }
    // ---- A = -strictLower(diag(beta) (K K^T * Gamma)) ----
    pair_matrix<C, DK, false>(sm, tid);
    __syncthreads();
    // ---- T - I by blocks, in place over A (strictly lower) ----
    invert_blocked<C, DK>(sm, tid);
    // The products below are warp MMAs (TF32 split three ways) on 16 x 8 tiles:
    // the C x 32 outputs (X, V', o) as C / 16 row blocks of four column tiles,
    // and the DK x 32 state slice as DK / 16 row blocks, each warp taking
    // consecutive tiles of one row block.
    constexpr int NTV = C / 32;    // column tiles per warp for C-row outputs
    constexpr int NTS = DK / 32;   // column tiles per warp for the state
    const int g8 = lane >> 2, t4 = lane & 3;
    const int vr0 = 16 * ((warp * NTV) / 4), vc0 = 8 * ((warp * NTV) % 4);  // this warp's C-row tiles
    // ---- X = diag(beta) (V - diag(exp(gcum)) K S) ----
    {
      float acc[NTV][4] = {};
      warp_mma_3xtf32<NTV>(acc, 0, DK,
                           [&](int m, int kk) { return KhT[swz<C>(kk, vr0 + m)]; },
                           [&](int kk, int n) { return S[kk * kDVS + vc0 + n]; }, g8, t4);
#pragma unroll
      for (int jj = 0; jj < NTV; ++jj)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int r = vr0 + g8 + 8 * (e >> 1), cc = vc0 + 8 * jj + 2 * t4 + (e & 1);
          const int64_t tk = c0 + r;
          const float vv = tk < seq_end ? to_f32(v[((size_t)tk * nv + h) * dv + cslice + cc]) : 0.f;
          V[r * kDVS + cc] = bt[r] * (vv - eg[r] * acc[jj][e]);
        }
    }
    __syncthreads();
    // ---- V' = T X = X + (T - I) X  (T - I is zero from the diagonal up) ----
    {
      float acc[NTV][4] = {};
      warp_mma_3xtf32<NTV>(acc, 0, vr0 + 16,
                           [&](int m, int kk) { return A[(vr0 + m) * L::AP + kk]; },
                           [&](int kk, int n) { return V[kk * kDVS + vc0 + n]; }, g8, t4);
      __syncthreads();  // every warp has read X
#pragma unroll
      for (int jj = 0; jj < NTV; ++jj)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int r = vr0 + g8 + 8 * (e >> 1), cc = vc0 + 8 * jj + 2 * t4 + (e & 1);
          V[r * kDVS + cc] += acc[jj][e];
        }
    }
    __syncthreads();
    // ---- P = (Q K^T * Gamma), lower including the diagonal ----
    pair_matrix<C, DK, true>(sm, tid);
    __syncthreads();
    // ---- o = diag(exp(gcum)) Q S + P V'  (P is zero above the diagonal) ----
    {
      float qs[NTV][4] = {}, pv[NTV][4] = {};
      warp_mma_3xtf32<NTV>(qs, 0, DK,
                           [&](int m, int kk) { return QhT[swz<C>(kk, vr0 + m)]; },
                           [&](int kk, int n) { return S[kk * kDVS + vc0 + n]; }, g8, t4);
      warp_mma_3xtf32<NTV>(pv, 0, vr0 + 16,
                           [&](int m, int kk) { return A[(vr0 + m) * L::AP + kk]; },
                           [&](int kk, int n) { return V[kk * kDVS + vc0 + n]; }, g8, t4);
#pragma unroll
      for (int jj = 0; jj < NTV; ++jj)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int r = vr0 + g8 + 8 * (e >> 1), cc = vc0 + 8 * jj + 2 * t4 + (e & 1);
          const int64_t tk = c0 + r;
          if (tk < seq_end)
            out[((size_t)tk * nv + h) * dv + cslice + cc] = from_f32<IO>(fmaf(eg[r], qs[jj][e], pv[jj][e]));
        }
    }
    __syncthreads();
    // ---- S <- exp(g_last) S + (K * exp(g_last - gcum))^T V' ----
    {
      const float decay = expf(gc[C - 1]);
      const int sr0 = 16 * ((warp * NTS) / 4), sc0 = 8 * ((warp * NTS) % 4);
      float acc[NTS][4] = {};
      warp_mma_3xtf32<NTS>(acc, 0, C,
                           [&](int m, int kk) { return KhT[swz<C>(sr0 + m, kk)]; },
                           [&](int kk, int n) { return ekl[kk] * V[kk * kDVS + sc0 + n]; }, g8, t4);
#pragma unroll
      for (int jj = 0; jj < NTS; ++jj)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int d = sr0 + g8 + 8 * (e >> 1), cc = sc0 + 8 * jj + 2 * t4 + (e & 1);
          S[d * kDVS + cc] = fmaf(S[d * kDVS + cc], decay, acc[jj][e]);
        }
    }
  }
  __syncthreads();
  if (a.s_final && srow >= 0) {
    for (int e = tid; e < DK * kDVS; e += kThreads) {
      const int d = e / kDVS, c = e % kDVS;
      a.s_final[state_off + (size_t)d * dv + cslice + c] = S[e];
    }
  }
}

template <int C, int DK, typename IO>
static cudaError_t launch_one(const ChunkArgs& a, cudaStream_t stream) {
  auto kern = chunk_fwd_simt_kernel<C, DK, IO>;
  const size_t smem = Smem<C, DK>::kBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(a.dv / kDVS, a.nv, a.num_seqs);
  kern<<<grid, kThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace simt

cudaError_t launch_chunk_simt(const ChunkArgs& a, int dk, int chunk, int io_bf16, cudaStream_t s) {
  using bf = __nv_bfloat16;
  if (dk == 64 && chunk == 64) return io_bf16 ? simt::launch_one<64, 64, bf>(a, s) : simt::launch_one<64, 64, float>(a, s);
  if (dk == 64 && chunk == 128) return io_bf16 ? simt::launch_one<128, 64, bf>(a, s) : simt::launch_one<128, 64, float>(a, s);
  if (dk == 128 && chunk == 64) return io_bf16 ? simt::launch_one<64, 128, bf>(a, s) : simt::launch_one<64, 128, float>(a, s);
  if (dk == 128 && chunk == 128) return io_bf16 ? simt::launch_one<128, 128, bf>(a, s) : simt::launch_one<128, 128, float>(a, s);
  return cudaErrorInvalidValue;
}

}  // namespace gdn

// decode_step.cu -- one-token gated delta rule step (decode), state updated in place.
//
// The token recurrence of the "手撕Qwen3-Next" walkthrough, section
// 一(一)5(2) (torch_recurrent_gated_delta_rule), for one token per sequence:
//
//   S <- alpha S (alpha = exp(g));  kv = S^T k_hat;  delta = beta (v - kv)
//   S <- S + k_hat delta^T;         o = S^T q_hat
//
// The state is read once and written once.  With the decayed old state
// D = alpha S_old, both reductions come from one pass over D:
//   kv_c = sum_r D[r,c] k_r,    o_c = sum_r D[r,c] q_r + delta_c (k_hat . q_hat)
// (the second is q^T (D + k delta^T)).  The kernel is bound by HBM: per
// (sequence, v-head) it streams Dk*Dv*4 bytes in and out.
//
// One CTA of 256 threads owns one (sequence, v-head).  Thread (rg, cg) holds
// 4 consecutive columns (one 16-byte vector) of DK/RG rows in registers, so
// every state byte is loaded with a 128-bit streaming load before any
// arithmetic starts and written back with a 128-bit streaming store.
//
// With the gated RMSNorm epilogue (kNorm; RMSNormGated of the walkthrough's
// sections 一(一)1 and 6) the Dv outputs of the row are normalised in the same
// CTA before the store: y = o / sqrt(mean(o^2) + eps) * w * silu(z).
//
// With the causal conv fused ahead of the step (kConv; section 一(一)3 and its
// torch_causal_conv1d_update) the CTA reads the packed projection [q | k | v]
// of its token and forms its q, k (qk-head j) and v (v-head h) channels as
// silu(bias + taps . [window, x]) itself, so q, k, v never reach memory.  The
// v channels' conv window belongs to this CTA alone and is updated by it.  The
// q, k channels are shared by the G = Nv / Nqk v-heads of the group: those G
// CTAs form a thread-block cluster, each arrives on the cluster barrier once it
// has read the old window, and rank 0 writes the new window after the wait.
#include "gdn_common.cuh"
#include "gdn_launch.h"

namespace gdn {
namespace decode {

constexpr int kThreads = 256;

// Relaxed arrive: what it must order are this CTA's reads of the shared windows,
// and their values have all been consumed (by the norms, before the block
// barrier) by the time any thread arrives.  A release arrive would also wait
// for the state loads still in flight.
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Conv + SiLU of channel c of sequence n (conv_state row `row`): returns the
// output, and leaves the window (K entries, oldest first) and the new input in
// win / xin for the state update.
template <typename IO>
__device__ __forceinline__ float conv_channel(const StepArgs& a, int n, int64_t row, int chans, int c,
                                              float (&win)[4], float& xin) {
  const int K = a.cks;
  const IO* st = static_cast<const IO*>(a.cstate) + ((size_t)row * chans + c) * K;
  xin = to_f32(static_cast<const IO*>(a.cx)[(size_t)n * chans + c]);
#pragma unroll
  for (int i = 0; i < 4; ++i) win[i] = i < K ? to_f32(st[i]) : 0.f;
  // taps 0..K-2 meet window entries 1..K-1, tap K-1 the new input
  float acc = a.cb ? a.cb[c] : 0.f;
#pragma unroll
  for (int i = 0; i + 1 < 4; ++i)
    if (i + 1 < K) acc = fmaf(a.cw[(size_t)c * K + i], win[i + 1], acc);
  return silu(fmaf(a.cw[(size_t)c * K + K - 1], xin, acc));
}
template <typename IO>
__device__ __forceinline__ void conv_store(const StepArgs& a, int64_t row, int chans, int c, const float (&win)[4],
                                           float xin) {
  const int K = a.cks;
  IO* st = static_cast<IO*>(a.cstate) + ((size_t)row * chans + c) * K;
#pragma unroll
  for (int i = 0; i < 4; ++i)
    if (i + 1 < K) st[i] = from_f32<IO>(win[i + 1]);
  st[K - 1] = from_f32<IO>(xin);
}

template <int DK, int DV, typename IO, bool kRawGate, bool kNorm, bool kConv>
__global__ void __launch_bounds__(kThreads, 2) recurrent_step_kernel(StepArgs a) {
  constexpr int CG = DV / 4;         // column groups of 4 fp32
  constexpr int RG = kThreads / CG;  // row groups
  constexpr int RPT = DK / RG;       // rows per thread
  static_assert(RPT >= 1 && DK % RG == 0, "shape");
  __shared__ float qh[DK], kh[DK];
  __shared__ float red_k[RG][DV], red_q[RG][DV];
  __shared__ __align__(16) float delta[DV];
  __shared__ float kq_s;
  __shared__ float gate_s[2];  // exp(g), beta
  __shared__ float nrm_s[DV / 32];  // per-warp sums of o^2 (kNorm)

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int h = blockIdx.x, n = blockIdx.y;
  const int j = h / (a.nv / a.nqk);
  const int cg = tid % CG, rg = tid / CG;

  const int64_t srow = state_row(a, n);
  if (srow < 0) {  // a padding sequence: zero output, no state
    for (int c = tid; c < DV; c += kThreads) static_cast<IO*>(a.out)[((size_t)n * a.nv + h) * DV + c] = from_f32<IO>(0.f);
    return;
  }
  if (tid == 64) {  // warp 2 is idle while warps 0-1 normalise q and k; issued before the state loads
    float gv, bv;
    load_gate_t<kRawGate>(a, (size_t)n * a.nv + h, h, gv, bv);
    gate_s[0] = expf(gv);
    gate_s[1] = bv;
  }
  float zc = 0.f, wc = 0.f, o_keep = 0.f;  // the norm's gate, gain and input of column tid (kNorm)
  if (kNorm && tid < DV) {
    zc = to_f32(static_cast<const IO*>(a.nz)[((size_t)n * a.nv + h) * DV + tid]);
    wc = a.nw[tid];
  }
  // fused conv: this thread's v channel (tid < DV) and, in warps 0-1, 4 q / k channels per lane
  const int chans = 2 * a.nqk * DK + a.nv * DV;
  float vwin[4], vx = 0.f, vconv = 0.f;
  float4* st = reinterpret_cast<float4*>(a.state + ((size_t)srow * a.nv + h) * (size_t)DK * DV);
  float4 s[RPT];
#pragma unroll
  for (int i = 0; i < RPT; ++i) s[i] = __ldcs(st + (size_t)(i * RG + rg) * CG + cg);
  // after the state loads are issued, so their latency overlaps the conv's
  if (kConv && tid < DV) vconv = conv_channel<IO>(a, n, srow, chans, 2 * a.nqk * DK + h * DV + tid, vwin, vx);


  // q_hat, k_hat (warp 0: q, warp 1: k)
  constexpr int PER = DK / 32;
  float qkwin[PER][4], qkx[PER];  // fused conv: the windows this lane read (rank 0 rewrites them)
  if (warp < 2) {
    float x[PER];
    float ss = 0.f;
    if constexpr (kConv) {
#pragma unroll
      for (int e = 0; e < PER; ++e) {
        const int c = (warp == 0 ? 0 : a.nqk * DK) + j * DK + lane * PER + e;
        x[e] = conv_channel<IO>(a, n, srow, chans, c, qkwin[e], qkx[e]);
        ss += x[e] * x[e];
      }
    } else {
      const IO* src = static_cast<const IO*>(warp == 0 ? a.q : a.k) + ((size_t)n * a.nqk + j) * DK;
#pragma unroll
      for (int e = 0; e < PER; ++e) {
        x[e] = to_f32(src[lane * PER + e]);
        ss += x[e] * x[e];
      }
    }
    ss = warp_sum(ss);
    float f = a.qk_l2norm ? 1.f / sqrtf(ss + kNormEps) : 1.f;
    if (warp == 0) f *= a.scale;
    float* dst = warp == 0 ? qh : kh;
#pragma unroll
    for (int e = 0; e < PER; ++e) dst[lane * PER + e] = x[e] * f;
  }
  __syncthreads();
  if constexpr (kConv) cluster_arrive_relaxed();  // this CTA has read the shared q / k windows
  const float alpha = gate_s[0], bta = gate_s[1];
  if (warp == 0) {
    float p = 0.f;
    for (int d = lane; d < DK; d += 32) p += qh[d] * kh[d];
    p = warp_sum(p);
    if (lane == 0) kq_s = p;
  }

  // partial reductions of the decayed state over this thread's rows
  float pk[4] = {0.f, 0.f, 0.f, 0.f}, pq[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int i = 0; i < RPT; ++i) {
    const int r = i * RG + rg;
    s[i].x *= alpha; s[i].y *= alpha; s[i].z *= alpha; s[i].w *= alpha;
    const float kr = kh[r], qr = qh[r];
    pk[0] = fmaf(s[i].x, kr, pk[0]); pk[1] = fmaf(s[i].y, kr, pk[1]);
    pk[2] = fmaf(s[i].z, kr, pk[2]); pk[3] = fmaf(s[i].w, kr, pk[3]);
    pq[0] = fmaf(s[i].x, qr, pq[0]); pq[1] = fmaf(s[i].y, qr, pq[1]);
    pq[2] = fmaf(s[i].z, qr, pq[2]); pq[3] = fmaf(s[i].w, qr, pq[3]);
  }
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    red_k[rg][cg * 4 + c] = pk[c];
    red_q[rg][cg * 4 + c] = pq[c];
  }
  __syncthreads();
  if (tid < DV) {
    const int c = tid;
    float kv = 0.f, qs = 0.f;
#pragma unroll
    for (int r = 0; r < RG; ++r) {
      kv += red_k[r][c];
      qs += red_q[r][c];
    }
    const size_t vo = ((size_t)n * a.nv + h) * DV + c;
    const float vin = kConv ? vconv : to_f32(static_cast<const IO*>(a.v)[vo]);
    const float dl = bta * (vin - kv);
    delta[c] = dl;
    const float o = fmaf(dl, kq_s, qs);
    if constexpr (kNorm) {
      const float ss = warp_sum(o * o);
      if (lane == 0) nrm_s[warp] = ss;
      o_keep = o;
    } else {
      static_cast<IO*>(a.out)[vo] = from_f32<IO>(o);
    }
  }
  __syncthreads();
  if constexpr (kNorm) {
    if (tid < DV) {
      float ss = 0.f;
#pragma unroll
      for (int w = 0; w < DV / 32; ++w) ss += nrm_s[w];
      const float inv = rsqrtf(ss * (1.f / DV) + a.neps);
      static_cast<IO*>(a.out)[((size_t)n * a.nv + h) * DV + tid] = from_f32<IO>(o_keep * inv * wc * silu(zc));
    }
  }
  const float4 dl = *reinterpret_cast<const float4*>(delta + cg * 4);
#pragma unroll
  for (int i = 0; i < RPT; ++i) {
    const float kr = kh[i * RG + rg];
    float4 o;
    o.x = fmaf(kr, dl.x, s[i].x); o.y = fmaf(kr, dl.y, s[i].y);
    o.z = fmaf(kr, dl.z, s[i].z); o.w = fmaf(kr, dl.w, s[i].w);
    __stcs(st + (size_t)(i * RG + rg) * CG + cg, o);
  }
  if constexpr (kConv) {
    if (tid < DV) conv_store<IO>(a, srow, chans, 2 * a.nqk * DK + h * DV + tid, vwin, vx);
    cluster_wait_acquire();  // every CTA of the group has read the old q / k windows
    if (warp < 2 && h % (a.nv / a.nqk) == 0) {
#pragma unroll
      for (int e = 0; e < PER; ++e)
        conv_store<IO>(a, srow, chans, (warp == 0 ? 0 : a.nqk * DK) + j * DK + lane * PER + e, qkwin[e], qkx[e]);
    }
  }
}

template <int DK, int DV, typename IO, bool kRaw, bool kNorm, bool kConv>
static cudaError_t launch_cfg(const StepArgs& a, cudaStream_t stream) {
  auto kernel = recurrent_step_kernel<DK, DV, IO, kRaw, kNorm, kConv>;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.nv, a.num_seqs);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  if (kConv) {  // the G v-heads of a qk group (consecutive in x) form one cluster
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = a.nv / a.nqk;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, a);
  return e != cudaSuccess ? e : cudaGetLastError();
}

template <int DK, int DV, typename IO, bool kRaw>
static cudaError_t launch_gate(const StepArgs& a, cudaStream_t s) {
  if (a.cx) return a.nz ? launch_cfg<DK, DV, IO, kRaw, true, true>(a, s) : launch_cfg<DK, DV, IO, kRaw, false, true>(a, s);
  return a.nz ? launch_cfg<DK, DV, IO, kRaw, true, false>(a, s) : launch_cfg<DK, DV, IO, kRaw, false, false>(a, s);
}

template <int DK, int DV, typename IO>
static cudaError_t launch_one(const StepArgs& a, cudaStream_t stream) {
  return a.A_log ? launch_gate<DK, DV, IO, true>(a, stream) : launch_gate<DK, DV, IO, false>(a, stream);
}

}  // namespace decode

cudaError_t launch_recurrent_step(const StepArgs& a, int dk, int dv, int io_bf16, cudaStream_t s) {
  using bf = __nv_bfloat16;
  if (dk == 64 && dv == 64) return io_bf16 ? decode::launch_one<64, 64, bf>(a, s) : decode::launch_one<64, 64, float>(a, s);
  if (dk == 64 && dv == 128) return io_bf16 ? decode::launch_one<64, 128, bf>(a, s) : decode::launch_one<64, 128, float>(a, s);
  if (dk == 128 && dv == 64) return io_bf16 ? decode::launch_one<128, 64, bf>(a, s) : decode::launch_one<128, 64, float>(a, s);
  if (dk == 128 && dv == 128) return io_bf16 ? decode::launch_one<128, 128, bf>(a, s) : decode::launch_one<128, 128, float>(a, s);
  return cudaErrorInvalidValue;
}

}  // namespace gdn

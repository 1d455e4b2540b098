// gdn_abi.cu -- the extern "C" boundary of libgdn.so: argument validation,
// kernel choice and launch on the caller's stream.  See include/gdn.h.
#include <cmath>
#include <cstdint>

#include "../../include/gdn.h"
#include "gdn_common.cuh"
#include "gdn_launch.h"

#define GDN_API extern "C" __attribute__((visibility("default")))

namespace {

constexpr int kMaxDevices = 64;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

struct Range {
  uintptr_t lo, hi;  // [lo, hi)
};

Range range_of(const void* p, size_t bytes) {
  const uintptr_t lo = reinterpret_cast<uintptr_t>(p);
  return Range{lo, lo + bytes};
}

bool overlap(Range a, Range b) {
  if (a.lo == a.hi || b.lo == b.hi) return false;
  return a.lo < b.hi && b.lo < a.hi;
}

// The device status word every kernel reports into (gdn::kStatus* bits), and
// the word gdn_device_status reads it into.  The kernels get the word's device
// address, looked up once per device (cudaGetSymbolAddress, current device).
__device__ unsigned int g_status_word;
__device__ unsigned int g_status_taken;

unsigned int* status_word() {
  static unsigned int* addr[kMaxDevices] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
    addr[dev] = static_cast<unsigned int*>(p);
  }
  return addr[dev];
}

// Reads and clears the status word in one atomic step, in stream order.
__global__ void take_status_kernel() { g_status_taken = atomicExch(&g_status_word, 0u); }

// The library ships sm_100a code only: require a compute capability 10.0 device.
int check_device() {
  static int ok[kMaxDevices] = {0};  // 0 unknown, 1 ok, -1 bad
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GDN_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return GDN_ERR_DEVICE;
  if (ok[dev] == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return GDN_ERR_CUDA;
    ok[dev] = (major == 10 && minor == 0) ? 1 : -1;
  }
  return ok[dev] == 1 ? GDN_OK : GDN_ERR_DEVICE;
}

int check_params(const gdn_params_t* p) {
  if (!p) return GDN_ERR_NULL;
  if (p->num_qk_heads < 1 || p->num_v_heads < 1 || p->num_v_heads > 65535 ||
      p->num_v_heads % p->num_qk_heads != 0)
    return GDN_ERR_SHAPE;
  if ((p->head_k_dim != 64 && p->head_k_dim != 128) || (p->head_v_dim != 64 && p->head_v_dim != 128))
    return GDN_ERR_SHAPE;
  if (p->io_dtype != GDN_DTYPE_F32 && p->io_dtype != GDN_DTYPE_BF16) return GDN_ERR_SHAPE;
  if (p->kernel < GDN_KERNEL_AUTO || p->kernel > GDN_KERNEL_TC) return GDN_ERR_SHAPE;
  if (!std::isfinite(p->scale)) return GDN_ERR_SHAPE;
  return GDN_OK;
}

float resolve_scale(const gdn_params_t* p) {
  return p->scale > 0.f ? p->scale : 1.0f / std::sqrt((float)p->head_k_dim);
}

}  // namespace

GDN_API int gdn_version(void) { return (1 << 16) | 6; }

GDN_API const char* gdn_status_string(int status) {
  switch (status) {
    case GDN_OK: return "GDN_OK";
    case GDN_ERR_NULL: return "GDN_ERR_NULL: a required pointer is NULL";
    case GDN_ERR_SHAPE: return "GDN_ERR_SHAPE: unsupported head count, head dim, chunk size or length";
    case GDN_ERR_ALIGN: return "GDN_ERR_ALIGN: a tensor pointer is not 16-byte aligned";
    case GDN_ERR_ALIAS: return "GDN_ERR_ALIAS: an output overlaps an input";
    case GDN_ERR_CUDA: return "GDN_ERR_CUDA: a CUDA call or kernel launch failed";
    case GDN_ERR_DEVICE: return "GDN_ERR_DEVICE: the current device is not compute capability 10.0";
    case GDN_ERR_DEVICE_TIMEOUT: return "GDN_ERR_DEVICE_TIMEOUT: a bounded in-kernel wait expired";
    case GDN_ERR_SEQLENS:
      return "GDN_ERR_SEQLENS: cu_seqlens was not non-decreasing from 0 to total_tokens (rows outside were skipped)";
    case GDN_ERR_GATE: return "GDN_ERR_GATE: a gate g > 0 or NaN reached the tensor-core kernel, which needs g <= 0";
    default: return "GDN: unknown status";
  }
}

// Validates the fusions of an extension block that do not depend on the call.
static int check_ext(const gdn_ext_t& x) {
  if ((x.A_log == nullptr) != (x.dt_bias == nullptr)) return GDN_ERR_NULL;
  if ((x.A_log && !aligned4(x.A_log)) || (x.dt_bias && !aligned4(x.dt_bias))) return GDN_ERR_ALIGN;
  if (x.slot_ids) {
    if (x.num_slots < 1) return GDN_ERR_SHAPE;
    if (!aligned4(x.slot_ids)) return GDN_ERR_ALIGN;
  }
  if (x.norm_z) {
    if (!x.norm_weight) return GDN_ERR_NULL;
    if (!std::isfinite(x.norm_eps) || x.norm_eps < 0.f) return GDN_ERR_SHAPE;
    if (!aligned16(x.norm_z) || !aligned16(x.norm_weight)) return GDN_ERR_ALIGN;
  }
  if (x.conv_x) {
    if (!x.conv_state || !x.conv_weight) return GDN_ERR_NULL;
    if (x.conv_kernel_size < 1 || x.conv_kernel_size > 4) return GDN_ERR_SHAPE;
    if (!aligned16(x.conv_x) || !aligned16(x.conv_state) || !aligned4(x.conv_weight) ||
        (x.conv_bias && !aligned4(x.conv_bias)))
      return GDN_ERR_ALIGN;
  }
  return GDN_OK;
}

// Every chunked-forward entry point lands here; `x` selects the fusions
// (fused gate: the g, beta slots hold the raw projections a, b; slot pool;
// gated RMSNorm epilogue).
static int chunk_fwd_impl(const void* q, const void* k, const void* v, const float* g,
                          const float* beta, const float* initial_state, const int32_t* cu_seqlens,
                          int32_t num_seqs, int64_t total_tokens, int32_t chunk_size, void* out,
                          float* final_state, const gdn_params_t* p, void* cuda_stream,
                          const gdn_ext_t& x) {
  int rc = check_params(p);
  if (rc) return rc;
  // with no tokens nothing is read or written but the states: the token tensors may be NULL
  if (total_tokens != 0 && (!q || !k || !v || !g || !beta || !out)) return GDN_ERR_NULL;
  rc = check_ext(x);
  if (rc) return rc;
  if (x.conv_x) return GDN_ERR_SHAPE;  // the prefill conv is gdn_qkv_conv_fwd
  const float *A_log = x.A_log, *dt_bias = x.dt_bias;
  const int32_t* slots = x.slot_ids;
  const int32_t num_slots = x.num_slots;
  if (num_seqs < 1 || num_seqs > 65535) return GDN_ERR_SHAPE;
  if (total_tokens < 0 || total_tokens >= (int64_t(1) << 31)) return GDN_ERR_SHAPE;
  if (chunk_size != 64 && chunk_size != 128) return GDN_ERR_SHAPE;
  if (!cu_seqlens && total_tokens % num_seqs != 0) return GDN_ERR_SHAPE;
  const void* ptrs[] = {q, k, v, g, beta, initial_state, cu_seqlens, out, final_state};
  for (const void* ptr : ptrs)
    if (ptr && !aligned16(ptr)) return GDN_ERR_ALIGN;

  const size_t T = (size_t)total_tokens, N = (size_t)num_seqs;
  const size_t esz = p->io_dtype == GDN_DTYPE_BF16 ? 2 : 4;
  const size_t dk = p->head_k_dim, dv = p->head_v_dim;
  const size_t nqk = p->num_qk_heads, nv = p->num_v_heads;
  const Range rq = range_of(q, T * nqk * dk * esz), rk = range_of(k, T * nqk * dk * esz);
  const Range rv = range_of(v, T * nv * dv * esz);
  const Range rg = range_of(g, T * nv * 4), rb = range_of(beta, T * nv * 4);
  const Range ra = A_log ? range_of(A_log, nv * 4) : Range{0, 0};
  const Range rd = dt_bias ? range_of(dt_bias, nv * 4) : Range{0, 0};
  const size_t rows = slots ? (size_t)num_slots : N;  // state rows
  const Range rs0 = initial_state ? range_of(initial_state, rows * nv * dk * dv * 4) : Range{0, 0};
  const Range rcu = cu_seqlens ? range_of(cu_seqlens, (N + 1) * 4) : Range{0, 0};
  const Range rsl = slots ? range_of(slots, N * 4) : Range{0, 0};
  const Range ro = range_of(out, T * nv * dv * esz);
  const Range rsf = final_state ? range_of(final_state, rows * nv * dk * dv * 4) : Range{0, 0};
  const Range rz = x.norm_z ? range_of(x.norm_z, T * nv * dv * esz) : Range{0, 0};
  const Range rw = x.norm_z ? range_of(x.norm_weight, dv * 4) : Range{0, 0};
  for (Range r : {rq, rk, rv, rg, rb, ra, rd, rs0, rcu, rsl, rsf, rz, rw})
    if (overlap(ro, r)) return GDN_ERR_ALIAS;
  for (Range r : {rq, rk, rv, rg, rb, ra, rd, rcu, rsl, rz, rw})
    if (overlap(rsf, r)) return GDN_ERR_ALIAS;
  if (final_state && initial_state && (const void*)final_state != (const void*)initial_state &&
      overlap(rsf, rs0))
    return GDN_ERR_ALIAS;

  rc = check_device();
  if (rc) return rc;
  unsigned int* status = status_word();
  if (!status) return GDN_ERR_CUDA;

  gdn::ChunkArgs a{};
  a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.A_log = A_log; a.dt_bias = dt_bias;
  a.s0 = initial_state; a.cu = cu_seqlens; a.out = out; a.s_final = final_state;
  a.slots = slots; a.num_slots = num_slots;
  a.uniform_len = cu_seqlens ? 0 : (int32_t)(total_tokens / num_seqs);
  a.num_seqs = num_seqs;
  a.total_tokens = total_tokens;
  a.status = status;
  a.nqk = p->num_qk_heads; a.nv = p->num_v_heads; a.dv = p->head_v_dim;
  a.qk_l2norm = p->qk_l2norm ? 1 : 0;
  a.scale = resolve_scale(p);
  a.nz = x.norm_z; a.nw = x.norm_weight; a.neps = x.norm_eps;
  cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);

  const int bf16 = p->io_dtype == GDN_DTYPE_BF16;
  const bool tc_ok = gdn::chunk_tc_supported(p->head_k_dim, p->head_v_dim, chunk_size, bf16);
  if (p->kernel == GDN_KERNEL_TC && !tc_ok) return GDN_ERR_SHAPE;
  // Both chunk kernels split Dv across CTAs and store o; the norm epilogue then
  // rewrites the rows in place (one HBM-bound pass).  Fused into the
  // tensor-core kernel's output warps it measured slower: those warps also
  // update rows 64..127 of the state, so their epilogue sits on the serial chain.
  a.nz = nullptr;
  cudaError_t e;
  // an empty batch reads no token and only carries the states over: the CUDA-core
  // launcher does that for every kernel setting
  if (tc_ok && p->kernel != GDN_KERNEL_SIMT && total_tokens > 0)
    e = gdn::launch_chunk_tc(a, total_tokens, stream);
  else
    e = gdn::launch_chunk_simt(a, p->head_k_dim, chunk_size, bf16, stream);
  if (e == cudaSuccess && x.norm_z)
    e = gdn::launch_gated_rmsnorm(out, x.norm_z, x.norm_weight, x.norm_eps, out, total_tokens * (int64_t)nv,
                                  (int)dv, bf16, stream);
  return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

static gdn_ext_t ext_of(const float* A_log, const float* dt_bias, const int32_t* slots, int32_t num_slots) {
  gdn_ext_t x{};
  x.A_log = A_log; x.dt_bias = dt_bias; x.slot_ids = slots; x.num_slots = num_slots;
  return x;
}

GDN_API int gdn_chunk_fwd(const void* q, const void* k, const void* v, const float* g,
                          const float* beta, const float* initial_state,
                          const int32_t* cu_seqlens, int32_t num_seqs, int64_t total_tokens,
                          int32_t chunk_size, void* out, float* final_state,
                          const gdn_params_t* p, void* cuda_stream) {
  return chunk_fwd_impl(q, k, v, g, beta, initial_state, cu_seqlens, num_seqs, total_tokens, chunk_size, out,
                        final_state, p, cuda_stream, ext_of(nullptr, nullptr, nullptr, 0));
}

GDN_API int gdn_chunk_fwd_slots(const void* q, const void* k, const void* v, const float* g,
                                const float* beta, float* state_pool, const int32_t* slot_ids,
                                int32_t num_slots, const int32_t* cu_seqlens, int32_t num_seqs,
                                int64_t total_tokens, int32_t chunk_size, void* out,
                                const gdn_params_t* p, void* cuda_stream) {
  if (!state_pool || !slot_ids) return GDN_ERR_NULL;
  return chunk_fwd_impl(q, k, v, g, beta, state_pool, cu_seqlens, num_seqs, total_tokens, chunk_size, out,
                        state_pool, p, cuda_stream, ext_of(nullptr, nullptr, slot_ids, num_slots));
}

GDN_API int gdn_chunk_fwd_gated(const void* q, const void* k, const void* v, const float* a,
                                const float* b, const float* A_log, const float* dt_bias,
                                const float* initial_state, const int32_t* cu_seqlens,
                                int32_t num_seqs, int64_t total_tokens, int32_t chunk_size,
                                void* out, float* final_state, const gdn_params_t* p,
                                void* cuda_stream) {
  if (!A_log || !dt_bias) return GDN_ERR_NULL;
  return chunk_fwd_impl(q, k, v, a, b, initial_state, cu_seqlens, num_seqs, total_tokens, chunk_size, out,
                        final_state, p, cuda_stream, ext_of(A_log, dt_bias, nullptr, 0));
}

GDN_API int gdn_chunk_fwd_ex(const void* q, const void* k, const void* v, const float* g,
                             const float* beta, const float* initial_state, const int32_t* cu_seqlens,
                             int32_t num_seqs, int64_t total_tokens, int32_t chunk_size, void* out,
                             float* final_state, const gdn_params_t* p, const gdn_ext_t* ext,
                             void* cuda_stream) {
  const gdn_ext_t x = ext ? *ext : gdn_ext_t{};
  if (x.slot_ids && (!initial_state || final_state != initial_state)) return GDN_ERR_NULL;
  return chunk_fwd_impl(q, k, v, g, beta, initial_state, cu_seqlens, num_seqs, total_tokens, chunk_size, out,
                        final_state, p, cuda_stream, x);
}

static int recurrent_step_impl(const void* q, const void* k, const void* v, const float* g,
                               const float* beta, float* state, void* out, int32_t num_seqs,
                               const gdn_params_t* p, void* cuda_stream, const gdn_ext_t& x) {
  int rc = check_params(p);
  if (rc) return rc;
  rc = check_ext(x);
  if (rc) return rc;
  const bool conv = x.conv_x != nullptr;
  if (conv) {
    if (q || k || v) return GDN_ERR_SHAPE;  // the fused conv produces them
    if (p->num_v_heads / p->num_qk_heads > 8) return GDN_ERR_SHAPE;  // one cluster per qk group
  } else if (!q || !k || !v) {
    return GDN_ERR_NULL;
  }
  if (!g || !beta || !state || !out) return GDN_ERR_NULL;
  const float *A_log = x.A_log, *dt_bias = x.dt_bias;
  const int32_t* slots = x.slot_ids;
  const int32_t num_slots = x.num_slots;
  if (num_seqs < 1 || num_seqs > 65535) return GDN_ERR_SHAPE;
  const void* ptrs[] = {q, k, v, g, beta, state, out};
  for (const void* ptr : ptrs)
    if (ptr && !aligned16(ptr)) return GDN_ERR_ALIGN;
  const size_t N = (size_t)num_seqs;
  const size_t esz = p->io_dtype == GDN_DTYPE_BF16 ? 2 : 4;
  const size_t dk = p->head_k_dim, dv = p->head_v_dim;
  const size_t nqk = p->num_qk_heads, nv = p->num_v_heads;
  const Range rq = range_of(q, N * nqk * dk * esz), rk = range_of(k, N * nqk * dk * esz);
  const Range rv = range_of(v, N * nv * dv * esz);
  const Range rg = range_of(g, N * nv * 4), rb = range_of(beta, N * nv * 4);
  const Range ra = A_log ? range_of(A_log, nv * 4) : Range{0, 0};
  const Range rd = dt_bias ? range_of(dt_bias, nv * 4) : Range{0, 0};
  const Range rs = range_of(state, (slots ? (size_t)num_slots : N) * nv * dk * dv * 4);
  const Range rsl = slots ? range_of(slots, N * 4) : Range{0, 0};
  const Range ro = range_of(out, N * nv * dv * esz);
  const Range rz = x.norm_z ? range_of(x.norm_z, N * nv * dv * esz) : Range{0, 0};
  const Range rw = x.norm_z ? range_of(x.norm_weight, dv * 4) : Range{0, 0};
  const size_t C = 2 * nqk * dk + nv * dv, CK = (size_t)x.conv_kernel_size;
  const Range rcx = conv ? range_of(x.conv_x, N * C * esz) : Range{0, 0};
  const Range rcs = conv ? range_of(x.conv_state, (slots ? (size_t)num_slots : N) * C * CK * esz) : Range{0, 0};
  const Range rcw = conv ? range_of(x.conv_weight, C * CK * 4) : Range{0, 0};
  const Range rcb = conv && x.conv_bias ? range_of(x.conv_bias, C * 4) : Range{0, 0};
  for (Range r : {rq, rk, rv, rg, rb, ra, rd, rs, rsl, rz, rw, rcx, rcs, rcw, rcb})
    if (overlap(ro, r)) return GDN_ERR_ALIAS;
  for (Range r : {rq, rk, rv, rg, rb, ra, rd, rsl, rz, rw, rcx, rcs, rcw, rcb})
    if (overlap(rs, r)) return GDN_ERR_ALIAS;
  for (Range r : {rg, rb, ra, rd, rsl, rz, rw, rcx, rcw, rcb})
    if (overlap(rcs, r)) return GDN_ERR_ALIAS;

  rc = check_device();
  if (rc) return rc;

  gdn::StepArgs a{};
  a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.A_log = A_log; a.dt_bias = dt_bias;
  a.state = state; a.out = out; a.slots = slots; a.num_slots = num_slots;
  a.num_seqs = num_seqs;
  a.nqk = p->num_qk_heads; a.nv = p->num_v_heads;
  a.qk_l2norm = p->qk_l2norm ? 1 : 0;
  a.scale = resolve_scale(p);
  a.nz = x.norm_z; a.nw = x.norm_weight; a.neps = x.norm_eps;
  a.cx = x.conv_x; a.cstate = x.conv_state; a.cw = x.conv_weight; a.cb = x.conv_bias;
  a.cks = x.conv_kernel_size;
  cudaError_t e = gdn::launch_recurrent_step(a, p->head_k_dim, p->head_v_dim,
                                             p->io_dtype == GDN_DTYPE_BF16,
                                             static_cast<cudaStream_t>(cuda_stream));
  return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

GDN_API int gdn_recurrent_step(const void* q, const void* k, const void* v, const float* g,
                               const float* beta, float* state, void* out, int32_t num_seqs,
                               const gdn_params_t* p, void* cuda_stream) {
  return recurrent_step_impl(q, k, v, g, beta, state, out, num_seqs, p, cuda_stream,
                             ext_of(nullptr, nullptr, nullptr, 0));
}

GDN_API int gdn_recurrent_step_slots(const void* q, const void* k, const void* v, const float* g,
                                     const float* beta, float* state_pool, const int32_t* slot_ids,
                                     int32_t num_slots, void* out, int32_t num_seqs,
                                     const gdn_params_t* p, void* cuda_stream) {
  if (!slot_ids) return GDN_ERR_NULL;
  return recurrent_step_impl(q, k, v, g, beta, state_pool, out, num_seqs, p, cuda_stream,
                             ext_of(nullptr, nullptr, slot_ids, num_slots));
}

GDN_API int gdn_recurrent_step_gated(const void* q, const void* k, const void* v, const float* a,
                                     const float* b, const float* A_log, const float* dt_bias,
                                     float* state, void* out, int32_t num_seqs,
                                     const gdn_params_t* p, void* cuda_stream) {
  if (!A_log || !dt_bias) return GDN_ERR_NULL;
  return recurrent_step_impl(q, k, v, a, b, state, out, num_seqs, p, cuda_stream,
                             ext_of(A_log, dt_bias, nullptr, 0));
}

GDN_API int gdn_recurrent_step_ex(const void* q, const void* k, const void* v, const float* g,
                                  const float* beta, float* state, void* out, int32_t num_seqs,
                                  const gdn_params_t* p, const gdn_ext_t* ext, void* cuda_stream) {
  return recurrent_step_impl(q, k, v, g, beta, state, out, num_seqs, p, cuda_stream,
                             ext ? *ext : gdn_ext_t{});
}

GDN_API int gdn_gated_rmsnorm(const void* o, const void* z, const float* weight, float eps, void* y,
                              int64_t rows, int32_t dim, int32_t io_dtype, void* cuda_stream) {
  if (rows < 0 || rows >= (int64_t(1) << 31) || (dim != 64 && dim != 128)) return GDN_ERR_SHAPE;
  if (io_dtype != GDN_DTYPE_F32 && io_dtype != GDN_DTYPE_BF16) return GDN_ERR_SHAPE;
  if (!std::isfinite(eps) || eps < 0.f) return GDN_ERR_SHAPE;
  if (rows == 0) return GDN_OK;  // nothing is read or written
  if (!o || !z || !weight || !y) return GDN_ERR_NULL;
  for (const void* ptr : {o, z, (const void*)weight, (const void*)y})
    if (!aligned16(ptr)) return GDN_ERR_ALIGN;
  const size_t bytes = (size_t)rows * dim * (io_dtype == GDN_DTYPE_BF16 ? 2 : 4);
  const Range ry = range_of(y, bytes);
  if (overlap(ry, range_of(z, bytes)) || overlap(ry, range_of(weight, (size_t)dim * 4))) return GDN_ERR_ALIAS;
  if (y != o && overlap(ry, range_of(o, bytes))) return GDN_ERR_ALIAS;
  const int rc = check_device();
  if (rc) return rc;
  const cudaError_t e = gdn::launch_gated_rmsnorm(o, z, weight, eps, y, rows, dim, io_dtype == GDN_DTYPE_BF16,
                                                  static_cast<cudaStream_t>(cuda_stream));
  return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

// Shared validation of the two conv calls; fills the launch block.
static int conv_common(const void* x, const float* weight, const float* bias, int32_t kernel_size, void* q,
                       void* k, void* v, int32_t num_seqs, int64_t rows, const gdn_params_t* p, gdn::ConvArgs& a) {
  int rc = check_params(p);
  if (rc) return rc;
  if (!weight) return GDN_ERR_NULL;
  if (rows != 0 && (!x || !q || !k || !v)) return GDN_ERR_NULL;  // no rows: the tensors may be NULL
  if (kernel_size < 1 || kernel_size > 4) return GDN_ERR_SHAPE;
  if (num_seqs < 1 || num_seqs > 65535) return GDN_ERR_SHAPE;
  for (const void* ptr : {x, (const void*)q, (const void*)k, (const void*)v})
    if (ptr && !aligned16(ptr)) return GDN_ERR_ALIGN;
  if (!aligned16(weight) || (bias && !aligned4(bias))) return GDN_ERR_ALIGN;  // taps move as 16-byte vectors
  a = gdn::ConvArgs{};
  a.x = x; a.weight = weight; a.bias = bias; a.num_seqs = num_seqs; a.ksize = kernel_size;
  a.nqk = p->num_qk_heads; a.nv = p->num_v_heads; a.dk = p->head_k_dim; a.dv = p->head_v_dim;
  a.channels = 2 * a.nqk * a.dk + a.nv * a.dv;
  a.q = q; a.k = k; a.v = v;
  return GDN_OK;
}

GDN_API int gdn_qkv_conv_fwd(const void* mixed_qkv, const float* weight, const float* bias,
                             const void* conv_state_in, const int32_t* cu_seqlens, int32_t num_seqs,
                             int64_t total_tokens, int32_t kernel_size, void* q, void* k, void* v,
                             void* conv_state_out, const gdn_params_t* p, void* cuda_stream) {
  gdn::ConvArgs a;
  if (total_tokens < 0 || total_tokens >= (int64_t(1) << 31)) return GDN_ERR_SHAPE;
  int rc = conv_common(mixed_qkv, weight, bias, kernel_size, q, k, v, num_seqs, total_tokens, p, a);
  if (rc) return rc;
  if (!cu_seqlens && total_tokens % num_seqs != 0) return GDN_ERR_SHAPE;
  for (const void* ptr : {conv_state_in, (const void*)conv_state_out, (const void*)cu_seqlens})
    if (ptr && !aligned16(ptr)) return GDN_ERR_ALIGN;
  const size_t T = (size_t)total_tokens, N = (size_t)num_seqs, C = (size_t)a.channels, K = kernel_size;
  const size_t esz = p->io_dtype == GDN_DTYPE_BF16 ? 2 : 4;
  const Range rx = range_of(mixed_qkv, T * C * esz), rw = range_of(weight, C * K * 4);
  const Range rb = bias ? range_of(bias, C * 4) : Range{0, 0};
  const Range rsi = conv_state_in ? range_of(conv_state_in, N * C * K * esz) : Range{0, 0};
  const Range rcu = cu_seqlens ? range_of(cu_seqlens, (N + 1) * 4) : Range{0, 0};
  const size_t qkb = T * a.nqk * a.dk * esz;
  const Range rq = range_of(q, qkb), rk = range_of(k, qkb), rv = range_of(v, T * a.nv * a.dv * esz);
  const Range rso = conv_state_out ? range_of(conv_state_out, N * C * K * esz) : Range{0, 0};
  for (Range o : {rq, rk, rv, rso})
    for (Range i : {rx, rw, rb, rcu})
      if (overlap(o, i)) return GDN_ERR_ALIAS;
  if (overlap(rq, rk) || overlap(rq, rv) || overlap(rk, rv) || overlap(rso, rq) || overlap(rso, rk) ||
      overlap(rso, rv))
    return GDN_ERR_ALIAS;
  for (Range o : {rq, rk, rv})
    if (overlap(o, rsi)) return GDN_ERR_ALIAS;
  if (conv_state_out && conv_state_in && conv_state_out != conv_state_in && overlap(rso, rsi))
    return GDN_ERR_ALIAS;
  rc = check_device();
  if (rc) return rc;
  a.status = status_word();
  if (!a.status) return GDN_ERR_CUDA;
  a.state_in = conv_state_in; a.state_out = conv_state_out; a.cu = cu_seqlens;
  a.uniform_len = cu_seqlens ? 0 : (int32_t)(total_tokens / num_seqs);
  a.total_tokens = total_tokens;
  const cudaError_t e = gdn::launch_conv_fwd(a, p->io_dtype == GDN_DTYPE_BF16, static_cast<cudaStream_t>(cuda_stream));
  return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

GDN_API int gdn_qkv_conv_update(const void* mixed_qkv, const float* weight, const float* bias, void* conv_state,
                                const int32_t* slot_ids, int32_t num_slots, int32_t num_seqs,
                                int32_t kernel_size, void* q, void* k, void* v, const gdn_params_t* p,
                                void* cuda_stream) {
  gdn::ConvArgs a;
  int rc = conv_common(mixed_qkv, weight, bias, kernel_size, q, k, v, num_seqs, num_seqs, p, a);
  if (rc) return rc;
  if (!conv_state) return GDN_ERR_NULL;
  if (!aligned16(conv_state)) return GDN_ERR_ALIGN;
  if (slot_ids) {
    if (num_slots < 1) return GDN_ERR_SHAPE;
    if (!aligned4(slot_ids)) return GDN_ERR_ALIGN;
  }
  const size_t N = (size_t)num_seqs, C = (size_t)a.channels, K = kernel_size;
  const size_t esz = p->io_dtype == GDN_DTYPE_BF16 ? 2 : 4;
  const size_t rows = slot_ids ? (size_t)num_slots : N;
  const Range rx = range_of(mixed_qkv, N * C * esz), rw = range_of(weight, C * K * 4);
  const Range rb = bias ? range_of(bias, C * 4) : Range{0, 0};
  const Range rsl = slot_ids ? range_of(slot_ids, N * 4) : Range{0, 0};
  const Range rs = range_of(conv_state, rows * C * K * esz);
  const size_t qkb = N * a.nqk * a.dk * esz;
  const Range rq = range_of(q, qkb), rk = range_of(k, qkb), rv = range_of(v, N * a.nv * a.dv * esz);
  for (Range o : {rq, rk, rv, rs})
    for (Range i : {rx, rw, rb, rsl})
      if (overlap(o, i)) return GDN_ERR_ALIAS;
  if (overlap(rq, rk) || overlap(rq, rv) || overlap(rk, rv) || overlap(rs, rq) || overlap(rs, rk) ||
      overlap(rs, rv))
    return GDN_ERR_ALIAS;
  rc = check_device();
  if (rc) return rc;
  a.status = status_word();
  if (!a.status) return GDN_ERR_CUDA;
  a.state_in = conv_state; a.state_out = conv_state; a.slots = slot_ids; a.num_slots = num_slots;
  a.total_tokens = num_seqs;
  const cudaError_t e =
      gdn::launch_conv_update(a, p->io_dtype == GDN_DTYPE_BF16, static_cast<cudaStream_t>(cuda_stream));
  return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

GDN_API int gdn_selftest_wait_timeout(int64_t limit_us, void* cuda_stream) {
  if (limit_us < 1 || limit_us > 2000000) return GDN_ERR_SHAPE;
  const int rc = check_device();
  if (rc) return rc;
  unsigned int* status = status_word();
  if (!status) return GDN_ERR_CUDA;
  const cudaError_t e =
      gdn::launch_selftest_wait((uint64_t)limit_us * 1000u, status, static_cast<cudaStream_t>(cuda_stream));
  return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

GDN_API int gdn_device_status(void* cuda_stream) {
  const int rc = check_device();
  if (rc) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  // read-and-clear on the device, in stream order, so that no report made
  // between a read and a separate clear is lost
  take_status_kernel<<<1, 1, 0, s>>>();
  if (cudaGetLastError() != cudaSuccess) return GDN_ERR_CUDA;
  unsigned int* taken = nullptr;
  if (cudaGetSymbolAddress(reinterpret_cast<void**>(&taken), g_status_taken) != cudaSuccess) return GDN_ERR_CUDA;
  unsigned int st = 0;
  if (cudaMemcpyAsync(&st, taken, sizeof(st), cudaMemcpyDeviceToHost, s) != cudaSuccess) return GDN_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return GDN_ERR_CUDA;
  if (st & gdn::kStatusTimeout) return GDN_ERR_DEVICE_TIMEOUT;
  if (st & gdn::kStatusSeqlens) return GDN_ERR_SEQLENS;
  if (st & gdn::kStatusGate) return GDN_ERR_GATE;
  return GDN_OK;
}

// sage_lib.cu - the C ABI (include/sage.h): argument validation, TMA tensor-map
// encoding and kernel launches.  One translation unit holds every kernel so the
// device watchdog word is a single symbol.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstring>
#include <mutex>
#include <type_traits>

#include "../../include/sage.h"
#include "attn_fwd.cuh"
#include "debug_qk.cuh"
#include "quant.cuh"
#include "sage_device.cuh"
#include "seq_table.cuh"

using namespace sage;

namespace {

constexpr size_t kMinAttnSmem = 116 * 1024;  // keeps the attention kernel at one CTA per SM

inline size_t round_up(size_t x, size_t m) { return (x + m - 1) / m * m; }

struct Layout {
  bool varlen = false;
  int nseq = 0;
  int64_t t_pad = 0;
  SeqDense dense{};
  SeqVarlen* var = nullptr;  // points into caller-provided storage
};

// Validate the problem and compute the padded token layout.
sage_status_t plan(const sage_problem_t* p, Layout& L, SeqVarlen* storage) {
  if (p == nullptr) return SAGE_ERR_INVALID_ARGUMENT;
  if (p->batch < 1 || p->heads_q < 1 || p->heads_kv < 1) return SAGE_ERR_INVALID_ARGUMENT;
  if (p->heads_q % p->heads_kv != 0) return SAGE_ERR_INVALID_ARGUMENT;
  if (p->head_dim != 64 && p->head_dim != 128) return SAGE_ERR_UNSUPPORTED;
  if (p->dtype != SAGE_FP16 && p->dtype != SAGE_BF16) return SAGE_ERR_UNSUPPORTED;
  L.nseq = p->batch;
  if (p->cu_seqlens_host == nullptr) {
    if (p->seqlen < 1) return SAGE_ERR_INVALID_ARGUMENT;
    L.varlen = false;
    L.dense.nseq = p->batch;
    L.dense.len = p->seqlen;
    L.dense.pad_len = static_cast<int>(round_up(p->seqlen, kPad));
    L.t_pad = static_cast<int64_t>(L.dense.pad_len) * p->batch;
  } else {
    if (p->batch > kMaxSeq) return SAGE_ERR_INVALID_ARGUMENT;
    const int32_t* cu = p->cu_seqlens_host;
    if (cu[0] != 0) return SAGE_ERR_INVALID_ARGUMENT;
    int64_t tp = 0;
    for (int b = 0; b < p->batch; ++b) {
      if (cu[b + 1] < cu[b]) return SAGE_ERR_INVALID_ARGUMENT;
      tp += static_cast<int64_t>(round_up(cu[b + 1] - cu[b], kPad));
    }
    if (cu[p->batch] < 1) return SAGE_ERR_INVALID_ARGUMENT;
    L.varlen = true;
    L.t_pad = tp;
    if (storage != nullptr) {
      std::memset(storage, 0, sizeof(SeqVarlen));
      storage->nseq = p->batch;
      storage->t_pad = static_cast<int>(tp);
      int64_t off = 0, cta = 0;
      for (int b = 0; b <= p->batch; ++b) {
        storage->cu[b] = cu[b];
        storage->poff[b] = static_cast<int32_t>(off);
        storage->cta[b] = static_cast<int32_t>(cta);
        if (b < p->batch) {
          const int n = cu[b + 1] - cu[b];
          const int tiles = (n + kBlkQ - 1) / kBlkQ;  // one attention CTA per 128-row Q tile
          off += static_cast<int64_t>(round_up(n, kPad));
          cta += static_cast<int64_t>(p->heads_q) * tiles;
        }
      }
      L.var = storage;
    }
  }
  L.dense.t_pad = static_cast<int>(L.t_pad);
  // row coordinates of the TMA maps and element offsets must fit in 32 bits
  if (L.t_pad * static_cast<int64_t>(p->heads_q) >= (int64_t{1} << 31)) return SAGE_ERR_UNSUPPORTED;
  return SAGE_OK;
}

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

bool strides_ok(const sage_problem_t* p, const int64_t s[3], int elem_bytes) {
  if (s == nullptr) return false;
  const bool dense = p->cu_seqlens_host == nullptr;
  for (int i = dense ? 0 : 1; i < 3; ++i)
    if (s[i] <= 0 || (s[i] * elem_bytes) % 16 != 0) return false;
  return true;
}

sage_status_t device_ok() {
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SAGE_ERR_CUDA;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return SAGE_ERR_CUDA;
  return (major == 10 && minor == 0) ? SAGE_OK : SAGE_ERR_UNSUPPORTED;
}

sage_status_t launched() {
  return cudaGetLastError() == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// 2D uint8 tensor map: `inner` bytes per row, `rows` rows `pitch` bytes apart,
// boxes of box_inner x box_rows with the given swizzle.
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t pitch,
              uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle swz) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {pitch};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

CUtensorMapSwizzle qk_swizzle(int d) {
  return d == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
}

// ------------------------------------------------------------------ quant launches
template <typename T, int D, class Seq>
sage_status_t launch_quant_qk(const Seq& seq, const sage_problem_t* p, int64_t t_pad,
                              const void* q, const int64_t* qs, const void* k, const int64_t* ks,
                              int8_t* q8, float* q_scale, int8_t* k8, float* k_scale,
                              float* k_mean, void* ws, cudaStream_t st) {
  double* partial = reinterpret_cast<double*>(ws);
  const int nblk = static_cast<int>(t_pad / kPad);
  k_colsum_kernel<T, D, Seq><<<dim3(nblk, p->heads_kv), kQuantThreads, 0, st>>>(
      seq, reinterpret_cast<const T*>(k), ks[0], ks[1], ks[2], partial);
  k_mean_kernel<D, Seq><<<dim3(p->batch, p->heads_kv), D, 0, st>>>(seq, partial, p->heads_kv, k_mean);
  QKQuantArgs a{};
  a.q = q; a.k = k;
  a.qsb = qs[0]; a.qsh = qs[1]; a.qst = qs[2];
  a.ksb = ks[0]; a.ksh = ks[1]; a.kst = ks[2];
  a.q8 = q8; a.q_scale = q_scale; a.k8 = k8; a.k_scale = k_scale; a.k_mean = k_mean;
  a.hq = p->heads_q; a.hkv = p->heads_kv;
  a.nq_blocks = static_cast<int>(p->heads_q * (t_pad / kBlkQ));
  const int nk_blocks = static_cast<int>(p->heads_kv * (t_pad / kBlkK));
  quant_qk_kernel<T, D, Seq><<<a.nq_blocks + nk_blocks, kQuantThreads, 0, st>>>(seq, a);
  return launched();
}

template <typename T, int D, class Seq>
sage_status_t launch_quant_v(const Seq& seq, const sage_problem_t* p, int64_t t_pad, const void* v,
                             const int64_t* vs, uint8_t* v8, float* v_scale, void* ws,
                             cudaStream_t st) {
  const int nblk = static_cast<int>(t_pad / kPad);
  float* partial = reinterpret_cast<float*>(ws);
  float* vmax = partial + static_cast<size_t>(p->heads_kv) * nblk * D;
  v_colmax_kernel<T, D, Seq><<<dim3(nblk, p->heads_kv), kQuantThreads, 0, st>>>(
      seq, reinterpret_cast<const T*>(v), vs[0], vs[1], vs[2], partial);
  v_finalize_kernel<D, Seq><<<dim3(p->batch, p->heads_kv), D, 0, st>>>(seq, partial, p->heads_kv,
                                                                        vmax, v_scale);
  VQuantArgs a{};
  a.v = v; a.sb = vs[0]; a.sh = vs[1]; a.st = vs[2]; a.vmax = vmax; a.v8 = v8; a.hkv = p->heads_kv;
  quant_v_kernel<T, D, Seq><<<dim3(nblk, p->heads_kv), kQuantThreads, 0, st>>>(seq, a);
  return launched();
}

template <int D, class Seq>
sage_status_t launch_attn(const Seq& seq, int64_t ncta, const CUtensorMap& mq, const CUtensorMap& mk,
                          const CUtensorMap& mv, const AttnArgs& a, cudaStream_t st) {
  auto kern = sage_attn_fwd_kernel<D, Seq>;
  // the warpgroups trade registers with setmaxnreg; the split only adds up if the
  // kernel was compiled to exactly the launch allocation it assumes
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return SAGE_ERR_CUDA;
  if (fa.numRegs != kAttnLaunchRegs || fa.maxThreadsPerBlock < kAttnThreads) return SAGE_ERR_UNSUPPORTED;
  const size_t smem = std::max(static_cast<size_t>(AttnSmem<D>::kAlloc), kMinAttnSmem);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return SAGE_ERR_CUDA;
  kern<<<static_cast<unsigned>(ncta), kAttnThreads, smem, st>>>(mq, mk, mv, seq, a);
  return launched();
}

}  // namespace

// ====================================================================== C ABI
extern "C" {

const char* sage_status_string(sage_status_t s) {
  switch (s) {
    case SAGE_OK: return "SAGE_OK";
    case SAGE_ERR_INVALID_ARGUMENT: return "SAGE_ERR_INVALID_ARGUMENT";
    case SAGE_ERR_UNSUPPORTED: return "SAGE_ERR_UNSUPPORTED";
    case SAGE_ERR_CUDA: return "SAGE_ERR_CUDA";
    case SAGE_ERR_DEVICE_TIMEOUT: return "SAGE_ERR_DEVICE_TIMEOUT";
    case SAGE_ERR_TOO_LARGE: return "SAGE_ERR_TOO_LARGE";
  }
  return "SAGE_ERR_UNKNOWN";
}

sage_status_t sage_buffer_sizes(const sage_problem_t* p, sage_sizes_t* sz) {
  if (sz == nullptr) return SAGE_ERR_INVALID_ARGUMENT;
  Layout L;
  const sage_status_t st = plan(p, L, nullptr);
  if (st != SAGE_OK) return st;
  const size_t d = p->head_dim, tp = static_cast<size_t>(L.t_pad);
  sz->t_pad = tp;
  sz->q8 = static_cast<size_t>(p->heads_q) * tp * d;
  sz->q_scale = static_cast<size_t>(p->heads_q) * (tp / kBlkQ) * sizeof(float);
  sz->k8 = static_cast<size_t>(p->heads_kv) * tp * d;
  sz->k_scale = static_cast<size_t>(p->heads_kv) * (tp / kBlkK) * sizeof(float);
  sz->k_mean = static_cast<size_t>(p->batch) * p->heads_kv * d * sizeof(float);
  sz->v8 = static_cast<size_t>(p->heads_kv) * d * tp;
  sz->v_scale = sz->k_mean;
  sz->workspace_qk = static_cast<size_t>(p->heads_kv) * (tp / kPad) * d * sizeof(double);
  sz->workspace_v = static_cast<size_t>(p->heads_kv) * (tp / kPad) * d * sizeof(float) +
                    static_cast<size_t>(p->batch) * p->heads_kv * d * sizeof(float);
  return SAGE_OK;
}

sage_status_t sage_quant_qk(const sage_problem_t* p, const void* q, const int64_t q_strides[3],
                            const void* k, const int64_t k_strides[3], int8_t* q8, float* q_scale,
                            int8_t* k8, float* k_scale, float* k_mean, void* workspace,
                            size_t workspace_bytes, sage_stream_t stream) {
  static thread_local SeqVarlen var;
  Layout L;
  sage_status_t st = plan(p, L, &var);
  if (st != SAGE_OK) return st;
  sage_sizes_t sz;
  sage_buffer_sizes(p, &sz);
  if (!q || !k || !q8 || !q_scale || !k8 || !k_scale || !k_mean || !workspace)
    return SAGE_ERR_INVALID_ARGUMENT;
  if (!aligned16(q) || !aligned16(k) || !aligned16(q8) || !aligned16(k8) || !aligned16(workspace))
    return SAGE_ERR_INVALID_ARGUMENT;
  if (!strides_ok(p, q_strides, 2) || !strides_ok(p, k_strides, 2)) return SAGE_ERR_INVALID_ARGUMENT;
  if (workspace_bytes < sz.workspace_qk) return SAGE_ERR_INVALID_ARGUMENT;
  if ((st = device_ok()) != SAGE_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
#define SAGE_QK(T, D)                                                                           \
  return L.varlen ? launch_quant_qk<T, D>(*L.var, p, L.t_pad, q, q_strides, k, k_strides, q8,    \
                                          q_scale, k8, k_scale, k_mean, workspace, s)            \
                  : launch_quant_qk<T, D>(L.dense, p, L.t_pad, q, q_strides, k, k_strides, q8,   \
                                          q_scale, k8, k_scale, k_mean, workspace, s)
  if (p->dtype == SAGE_FP16) {
    if (p->head_dim == 128) { SAGE_QK(__half, 128); } else { SAGE_QK(__half, 64); }
  } else {
    if (p->head_dim == 128) { SAGE_QK(__nv_bfloat16, 128); } else { SAGE_QK(__nv_bfloat16, 64); }
  }
#undef SAGE_QK
}

sage_status_t sage_quant_v(const sage_problem_t* p, const void* v, const int64_t v_strides[3],
                           uint8_t* v8, float* v_scale, void* workspace, size_t workspace_bytes,
                           sage_stream_t stream) {
  static thread_local SeqVarlen var;
  Layout L;
  sage_status_t st = plan(p, L, &var);
  if (st != SAGE_OK) return st;
  sage_sizes_t sz;
  sage_buffer_sizes(p, &sz);
  if (!v || !v8 || !v_scale || !workspace) return SAGE_ERR_INVALID_ARGUMENT;
  if (!aligned16(v) || !aligned16(v8) || !aligned16(workspace)) return SAGE_ERR_INVALID_ARGUMENT;
  if (!strides_ok(p, v_strides, 2)) return SAGE_ERR_INVALID_ARGUMENT;
  if (workspace_bytes < sz.workspace_v) return SAGE_ERR_INVALID_ARGUMENT;
  if ((st = device_ok()) != SAGE_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
#define SAGE_V(T, D)                                                                             \
  return L.varlen ? launch_quant_v<T, D>(*L.var, p, L.t_pad, v, v_strides, v8, v_scale, workspace, s) \
                  : launch_quant_v<T, D>(L.dense, p, L.t_pad, v, v_strides, v8, v_scale, workspace, s)
  if (p->dtype == SAGE_FP16) {
    if (p->head_dim == 128) { SAGE_V(__half, 128); } else { SAGE_V(__half, 64); }
  } else {
    if (p->head_dim == 128) { SAGE_V(__nv_bfloat16, 128); } else { SAGE_V(__nv_bfloat16, 64); }
  }
#undef SAGE_V
}

sage_status_t sage_attn_fwd(const sage_problem_t* p, const int8_t* q8, const float* q_scale,
                            const int8_t* k8, const float* k_scale, const uint8_t* v8,
                            const float* v_scale, float sm_scale, int is_causal, void* out,
                            sage_dtype_t out_dtype, const int64_t out_strides[3], float* lse,
                            sage_stream_t stream) {
  static thread_local SeqVarlen var;
  Layout L;
  sage_status_t st = plan(p, L, &var);
  if (st != SAGE_OK) return st;
  if (!q8 || !q_scale || !k8 || !k_scale || !v8 || !v_scale || !out) return SAGE_ERR_INVALID_ARGUMENT;
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(v8) || !aligned16(out))
    return SAGE_ERR_INVALID_ARGUMENT;
  if (out_dtype != SAGE_FP16 && out_dtype != SAGE_BF16 && out_dtype != SAGE_FP32)
    return SAGE_ERR_UNSUPPORTED;
  if (!strides_ok(p, out_strides, out_dtype == SAGE_FP32 ? 4 : 2)) return SAGE_ERR_INVALID_ARGUMENT;
  if (!(sm_scale == sm_scale) || std::isinf(sm_scale)) return SAGE_ERR_INVALID_ARGUMENT;
  if ((st = device_ok()) != SAGE_OK) return st;
  const int d = p->head_dim;
  const uint64_t tp = static_cast<uint64_t>(L.t_pad);
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q8, d, tp * p->heads_q, d, d, kBlkQ, qk_swizzle(d)) ||
      !make_map(&mk, k8, d, tp * p->heads_kv, d, d, kKvTile, qk_swizzle(d)) ||
      !make_map(&mv, v8, tp, static_cast<uint64_t>(p->heads_kv) * d, tp, kKvTile, d,
                CU_TENSOR_MAP_SWIZZLE_128B))
    return SAGE_ERR_CUDA;
  AttnArgs a{};
  a.q_scale = q_scale; a.k_scale = k_scale; a.v_scale = v_scale;
  a.out = out; a.out_dtype = static_cast<int>(out_dtype);
  a.osb = out_strides[0]; a.osh = out_strides[1]; a.ost = out_strides[2];
  a.lse = lse;
  a.hq = p->heads_q; a.hkv = p->heads_kv; a.group = p->heads_q / p->heads_kv;
  const float scale = sm_scale > 0.0f ? sm_scale : 1.0f / std::sqrt(static_cast<float>(d));
  a.scale_log2 = scale * kLog2E;
  a.causal = is_causal ? 1 : 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (L.varlen) {
    const int64_t ncta = L.var->cta[p->batch];
    if (ncta == 0) return SAGE_OK;
    return d == 128 ? launch_attn<128>(*L.var, ncta, mq, mk, mv, a, s)
                    : launch_attn<64>(*L.var, ncta, mq, mk, mv, a, s);
  }
  const int64_t tiles = (L.dense.len + kBlkQ - 1) / kBlkQ;
  const int64_t ncta = static_cast<int64_t>(p->batch) * p->heads_q * tiles;
  return d == 128 ? launch_attn<128>(L.dense, ncta, mq, mk, mv, a, s)
                  : launch_attn<64>(L.dense, ncta, mq, mk, mv, a, s);
}

sage_status_t sage_debug_qk_int32(const sage_problem_t* p, const int8_t* q8, const int8_t* k8,
                                  int seq, int head_q, int32_t* s_out, sage_stream_t stream) {
  static thread_local SeqVarlen var;
  Layout L;
  sage_status_t st = plan(p, L, &var);
  if (st != SAGE_OK) return st;
  if (!q8 || !k8 || !s_out || !aligned16(q8) || !aligned16(k8) || !aligned16(s_out))
    return SAGE_ERR_INVALID_ARGUMENT;
  if (seq < 0 || seq >= p->batch || head_q < 0 || head_q >= p->heads_q)
    return SAGE_ERR_INVALID_ARGUMENT;
  if ((st = device_ok()) != SAGE_OK) return st;
  const int d = p->head_dim;
  const int n = L.varlen ? L.var->cu[seq + 1] - L.var->cu[seq] : L.dense.len;
  const int off = L.varlen ? L.var->poff[seq] : seq * L.dense.pad_len;
  const int plen = static_cast<int>(round_up(n, kPad));
  if (plen == 0) return SAGE_OK;
  const uint64_t tp = static_cast<uint64_t>(L.t_pad);
  CUtensorMap mq, mk;
  if (!make_map(&mq, q8, d, tp * p->heads_q, d, d, kBlkQ, qk_swizzle(d)) ||
      !make_map(&mk, k8, d, tp * p->heads_kv, d, d, kBlkQ, qk_swizzle(d)))
    return SAGE_ERR_CUDA;
  const int hk = head_q / (p->heads_q / p->heads_kv);
  const int q_row0 = static_cast<int>(head_q * tp + off), k_row0 = static_cast<int>(hk * tp + off);
  const dim3 grid(plen / kBlkQ, plen / kBlkQ);
  const size_t smem = 2 * kBlkQ * d + 64 + 1024;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (d == 128) {
    cudaFuncSetAttribute(debug_qk_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    debug_qk_kernel<128><<<grid, 128, smem, s>>>(mq, mk, q_row0, k_row0, plen, s_out);
  } else {
    cudaFuncSetAttribute(debug_qk_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    debug_qk_kernel<64><<<grid, 128, smem, s>>>(mq, mk, q_row0, k_row0, plen, s_out);
  }
  return launched();
}

sage_status_t sage_poll_device_status(sage_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return SAGE_ERR_CUDA;
  uint32_t w = 0;
  if (cudaMemcpyFromSymbol(&w, g_watchdog, sizeof(w)) != cudaSuccess) return SAGE_ERR_CUDA;
  if (w == 0) return SAGE_OK;
  const uint32_t zero = 0;
  if (cudaMemcpyToSymbol(g_watchdog, &zero, sizeof(zero)) != cudaSuccess) return SAGE_ERR_CUDA;
  return SAGE_ERR_DEVICE_TIMEOUT;
}

}  // extern "C"

// ====================================================================== scratch-free sage_quant_qk
// sage_quant_qk writes per-block fp64 column sums of K into a workspace the caller
// allocates.  Some callers cannot allocate device memory at the moment they
// quantize: code running inside a framework hook whose caching allocator is
// locked or mid-teardown, plugins that may only touch the tensors they are handed,
// and pipelines whose every device buffer is reserved up front.  For them
// sage_quant_qk_noalloc takes that scratch from the array below instead.
//
// The array is a fixed, modest size held by every GPU that loads this library
// until the process exits; problems that need more are rejected.  Host code may
// not use the array's name as a device address (it is a host-side stand-in), so
// the device address is looked up with cudaGetSymbolAddress, once per device, on
// that device's first call.  All calls share the array and it keeps the last
// call's contents; every word a call reads was written earlier in the same call,
// so nothing needs clearing, but calls that overlap on the GPU race on it.
static __device__ __align__(256) unsigned char g_quant_qk_scratch[SAGE_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_quant_qk_scratch on the current device (looked up once).
sage_status_t static_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SAGE_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return SAGE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_quant_qk_scratch) != cudaSuccess || ptr == nullptr)
      return SAGE_ERR_CUDA;
    g_scratch_addr[dev] = ptr;
  }
  *out = g_scratch_addr[dev];
  return SAGE_OK;
}

}  // namespace

extern "C" sage_status_t sage_quant_qk_noalloc(const sage_problem_t* p, const void* q,
                                               const int64_t q_strides[3], const void* k,
                                               const int64_t k_strides[3], int8_t* q8,
                                               float* q_scale, int8_t* k8, float* k_scale,
                                               float* k_mean, sage_stream_t stream) {
  static thread_local SeqVarlen var;
  Layout L;
  sage_status_t st = plan(p, L, &var);
  if (st != SAGE_OK) return st;
  sage_sizes_t sz;
  sage_buffer_sizes(p, &sz);
  if (!q || !k || !q8 || !q_scale || !k8 || !k_scale || !k_mean) return SAGE_ERR_INVALID_ARGUMENT;
  if (!aligned16(q) || !aligned16(k) || !aligned16(q8) || !aligned16(k8))
    return SAGE_ERR_INVALID_ARGUMENT;
  if (!strides_ok(p, q_strides, 2) || !strides_ok(p, k_strides, 2)) return SAGE_ERR_INVALID_ARGUMENT;
  if (sz.workspace_qk > SAGE_NOALLOC_SCRATCH_BYTES) return SAGE_ERR_TOO_LARGE;
  if ((st = device_ok()) != SAGE_OK) return st;
  void* ws = nullptr;
  if ((st = static_scratch(&ws)) != SAGE_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
#define SAGE_QK(T, D)                                                                           \
  return L.varlen ? launch_quant_qk<T, D>(*L.var, p, L.t_pad, q, q_strides, k, k_strides, q8,    \
                                          q_scale, k8, k_scale, k_mean, ws, s)                   \
                  : launch_quant_qk<T, D>(L.dense, p, L.t_pad, q, q_strides, k, k_strides, q8,   \
                                          q_scale, k8, k_scale, k_mean, ws, s)
  if (p->dtype == SAGE_FP16) {
    if (p->head_dim == 128) { SAGE_QK(__half, 128); } else { SAGE_QK(__half, 64); }
  } else {
    if (p->head_dim == 128) { SAGE_QK(__nv_bfloat16, 128); } else { SAGE_QK(__nv_bfloat16, 64); }
  }
#undef SAGE_QK
}

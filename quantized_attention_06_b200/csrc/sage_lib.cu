// sage_lib.cu - the C ABI (include/sage.h): argument validation, TMA tensor-map
// encoding and kernel launches.  One translation unit holds every kernel so the
// device watchdog word is a single symbol.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstring>
#include <algorithm>
#include <mutex>
#include <type_traits>

#include "../../include/sage.h"
#include "attn_fwd.cuh"
#include "debug_qk.cuh"
#include "quant.cuh"
#include "quant_fused.cuh"
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
  if (p->granularity != SAGE_GRAN_BLOCK && p->granularity != SAGE_GRAN_THREAD)
    return SAGE_ERR_INVALID_ARGUMENT;
  if (p->pv != SAGE_PV_FP8 && p->pv != SAGE_PV_FP16) return SAGE_ERR_INVALID_ARGUMENT;
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
          // one attention CTA per pair of 128-row Q tiles
          const int pairs = ((n + kBlkQ - 1) / kBlkQ + 1) / 2;
          off += static_cast<int64_t>(round_up(n, kPad));
          cta += static_cast<int64_t>(p->heads_q) * pairs;
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

// The current device must be an sm_100 part, and `stream` must belong to it: the
// kernels run on the current device, so a stream of another device would make them
// dereference that device's pointers.
sage_status_t device_ok(sage_stream_t stream) {
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SAGE_ERR_CUDA;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return SAGE_ERR_CUDA;
  if (major != 10 || minor != 0) return SAGE_ERR_UNSUPPORTED;
  int sdev = -1;
  if (cudaStreamGetDevice(reinterpret_cast<cudaStream_t>(stream), &sdev) != cudaSuccess)
    return SAGE_ERR_CUDA;
  return sdev == dev ? SAGE_OK : SAGE_ERR_INVALID_ARGUMENT;
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
  a.fine = p->granularity == SAGE_GRAN_THREAD ? 1 : 0;
  const int nk_blocks = static_cast<int>(p->heads_kv * (t_pad / kBlkK));
  quant_qk_kernel<T, D, Seq><<<a.nq_blocks + nk_blocks, kQuantThreads, 0, st>>>(seq, a);
  return launched();
}

template <typename T, int D, class Seq>
sage_status_t launch_quant_v(const Seq& seq, const sage_problem_t* p, int64_t t_pad, const void* v,
                             const int64_t* vs, uint8_t* v8, float* v_scale, void* ws,
                             cudaStream_t st) {
  const int nblk = static_cast<int>(t_pad / kPad);
  if (p->pv == SAGE_PV_FP16) {  // V keeps its 16-bit values, transposed; unit scales
    VQuantArgs a{};
    a.v = v; a.sb = vs[0]; a.sh = vs[1]; a.st = vs[2]; a.v8 = v8; a.hkv = p->heads_kv;
    transpose_v16_kernel<T, D, Seq><<<dim3(nblk, p->heads_kv), kQuantThreads, 0, st>>>(seq, a);
    const int64_t ns = static_cast<int64_t>(p->batch) * p->heads_kv * D;
    fill_ones_kernel<<<static_cast<unsigned>((ns + 255) / 256), 256, 0, st>>>(v_scale, ns);
    return launched();
  }
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

template <int D, class Seq, bool kFine, int PV>
sage_status_t launch_attn(const Seq& seq, int64_t ncta, const CUtensorMap& mq, const CUtensorMap& mk,
                          const CUtensorMap& mv, const AttnArgs& a, cudaStream_t st) {
  auto kern = sage_attn_fwd_kernel<D, Seq, kFine, PV>;
  // the warpgroups trade registers with setmaxnreg; the split only adds up if the
  // kernel was compiled to exactly the launch allocation it assumes
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return SAGE_ERR_CUDA;
  if (fa.numRegs != kAttnLaunchRegs || fa.maxThreadsPerBlock < kAttnThreads) return SAGE_ERR_UNSUPPORTED;
  const size_t smem = std::max(static_cast<size_t>(AttnCfg<D, PV>::kAlloc), kMinAttnSmem);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return SAGE_ERR_CUDA;
  kern<<<static_cast<unsigned>(ncta), kAttnThreads, smem, st>>>(mq, mk, mv, seq, a);
  return launched();
}

// Template dispatch of the attention kernel: head dim, granularity, PV format.
template <class Seq>
sage_status_t dispatch_attn(const Seq& seq, int64_t ncta, int d, bool fine, int pv,
                            const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                            const AttnArgs& a, cudaStream_t st) {
#define SAGE_ATTN(DD, FF, PP) \
  if (d == DD && fine == FF && pv == PP) return launch_attn<DD, Seq, FF, PP>(seq, ncta, mq, mk, mv, a, st)
  SAGE_ATTN(128, false, kPvE4m3); SAGE_ATTN(128, true, kPvE4m3);
  SAGE_ATTN(64, false, kPvE4m3);  SAGE_ATTN(64, true, kPvE4m3);
  SAGE_ATTN(128, false, kPvF16);  SAGE_ATTN(128, true, kPvF16);
  SAGE_ATTN(64, false, kPvF16);   SAGE_ATTN(64, true, kPvF16);
  SAGE_ATTN(128, false, kPvBf16); SAGE_ATTN(128, true, kPvBf16);
  SAGE_ATTN(64, false, kPvBf16);  SAGE_ATTN(64, true, kPvBf16);
#undef SAGE_ATTN
  return SAGE_ERR_UNSUPPORTED;
}

// 4-D 16-bit tensor map over an input (d, tokens, heads, batch): the three outer
// dimensions in ascending stride order, boxes of 64 channels x 128 tokens (128-byte
// swizzle).  Reports where the token, head and batch dimensions landed.
bool make_input_map(CUtensorMap* m, const void* base, const sage_problem_t* p, int heads,
                    const int64_t s[3], int64_t ntok, int* dim_tok, int* dim_head, int* dim_batch) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  const bool dense = p->cu_seqlens_host == nullptr;
  struct Dim { uint64_t size, stride; int kind; } dm[3];
  dm[0] = {static_cast<uint64_t>(ntok), static_cast<uint64_t>(s[2]) * 2, 0};
  dm[1] = {static_cast<uint64_t>(heads), static_cast<uint64_t>(s[1]) * 2, 1};
  if (dense) {
    dm[2] = {static_cast<uint64_t>(p->batch), static_cast<uint64_t>(s[0]) * 2, 2};
  } else {  // packed sequences: a unit batch dimension beyond the whole tensor
    const uint64_t ext = std::max(dm[0].size * dm[0].stride, dm[1].size * dm[1].stride);
    dm[2] = {1, round_up(ext, 16), 2};
  }
  std::sort(dm, dm + 3, [](const Dim& x, const Dim& y) { return x.stride < y.stride; });
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(p->head_dim), dm[0].size, dm[1].size, dm[2].size};
  cuuint64_t strides[3] = {dm[0].stride, dm[1].stride, dm[2].stride};
  cuuint32_t box[4] = {64, 1, 1, 1}, estr[4] = {1, 1, 1, 1};
  for (int i = 0; i < 3; ++i) {
    if (dm[i].kind == 0) { *dim_tok = i + 1; box[i + 1] = kPad; }
    if (dm[i].kind == 1) *dim_head = i + 1;
    if (dm[i].kind == 2) *dim_batch = i + 1;
  }
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT16, 4, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename T, int D, class Seq>
sage_status_t launch_quant_fused(const Seq& seq, const CUtensorMap& mq, const CUtensorMap& mk,
                                 const CUtensorMap& mv, const FusedQuantArgs& a, cudaStream_t st) {
  auto kern = quant_fused_kernel<T, D, Seq>;
  const int smem = FusedCfg<D>::kAlloc;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return SAGE_ERR_CUDA;
  int dev = 0, nsm = 0, coop = 0, per_sm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kFusedThreads, smem) != cudaSuccess)
    return SAGE_ERR_CUDA;
  if (!coop || per_sm < 1) return SAGE_ERR_UNSUPPORTED;
  void* args[] = {const_cast<CUtensorMap*>(&mq), const_cast<CUtensorMap*>(&mk),
                  const_cast<CUtensorMap*>(&mv), const_cast<Seq*>(&seq),
                  const_cast<FusedQuantArgs*>(&a)};
  if (cudaLaunchCooperativeKernel(reinterpret_cast<void*>(kern), dim3(nsm), dim3(kFusedThreads), args,
                                  smem, st) != cudaSuccess)
    return SAGE_ERR_CUDA;
  return launched();
}

// Template dispatch: head dim, granularity, PV format (the sequence table type is the caller's).
template <class Seq>
sage_status_t dispatch_quant_fused(const Seq& seq, const sage_problem_t* p, const CUtensorMap& mq,
                                   const CUtensorMap& mk, const CUtensorMap& mv,
                                   const FusedQuantArgs& a, cudaStream_t st) {
  if (p->dtype == SAGE_FP16)
    return p->head_dim == 128 ? launch_quant_fused<__half, 128>(seq, mq, mk, mv, a, st)
                              : launch_quant_fused<__half, 64>(seq, mq, mk, mv, a, st);
  return p->head_dim == 128 ? launch_quant_fused<__nv_bfloat16, 128>(seq, mq, mk, mv, a, st)
                            : launch_quant_fused<__nv_bfloat16, 64>(seq, mq, mk, mv, a, st);
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
  const bool fine = p->granularity == SAGE_GRAN_THREAD;
  sz->q_scale = static_cast<size_t>(p->heads_q) * (tp / (fine ? 1 : kBlkQ)) * sizeof(float);
  sz->k8 = static_cast<size_t>(p->heads_kv) * tp * d;
  sz->k_scale = static_cast<size_t>(p->heads_kv) * (tp / (fine ? kBlkKFine : kBlkK)) * sizeof(float);
  sz->k_mean = static_cast<size_t>(p->batch) * p->heads_kv * d * sizeof(float);
  const bool pv16 = p->pv == SAGE_PV_FP16;
  sz->v8 = static_cast<size_t>(p->heads_kv) * d * tp * (pv16 ? 2 : 1);
  sz->v_scale = sz->k_mean;
  sz->workspace_qk = static_cast<size_t>(p->heads_kv) * (tp / kPad) * d * sizeof(double);
  sz->workspace_v = pv16 ? 0
                         : static_cast<size_t>(p->heads_kv) * (tp / kPad) * d * sizeof(float) +
                               static_cast<size_t>(p->batch) * p->heads_kv * d * sizeof(float);
  // fused: fp64 K partial sums, fp32 V partial maxima, fp32 vmax (offsets 256-aligned)
  sz->workspace_qkv = round_up(sz->workspace_qk, 256) +
                      round_up(static_cast<size_t>(p->heads_kv) * (tp / kPad) * d * sizeof(float), 256) +
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
  if ((st = device_ok(stream)) != SAGE_OK) return st;
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
  if (!v || !v8 || !v_scale || (!workspace && sz.workspace_v > 0)) return SAGE_ERR_INVALID_ARGUMENT;
  if (!aligned16(v) || !aligned16(v8) || !aligned16(workspace)) return SAGE_ERR_INVALID_ARGUMENT;
  if (!strides_ok(p, v_strides, 2)) return SAGE_ERR_INVALID_ARGUMENT;
  if (workspace_bytes < sz.workspace_v) return SAGE_ERR_INVALID_ARGUMENT;
  if ((st = device_ok(stream)) != SAGE_OK) return st;
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

sage_status_t sage_quant_qkv(const sage_problem_t* p, const void* q, const int64_t q_strides[3],
                             const void* k, const int64_t k_strides[3], const void* v,
                             const int64_t v_strides[3], int8_t* q8, float* q_scale, int8_t* k8,
                             float* k_scale, float* k_mean, void* v8, float* v_scale,
                             void* workspace, size_t workspace_bytes, sage_stream_t stream) {
  static thread_local SeqVarlen var;
  Layout L;
  sage_status_t st = plan(p, L, &var);
  if (st != SAGE_OK) return st;
  sage_sizes_t sz;
  sage_buffer_sizes(p, &sz);
  if (!q || !k || !v || !q8 || !q_scale || !k8 || !k_scale || !k_mean || !v8 || !v_scale || !workspace)
    return SAGE_ERR_INVALID_ARGUMENT;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(q8) || !aligned16(k8) ||
      !aligned16(v8) || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return SAGE_ERR_INVALID_ARGUMENT;
  if (!strides_ok(p, q_strides, 2) || !strides_ok(p, k_strides, 2) || !strides_ok(p, v_strides, 2))
    return SAGE_ERR_INVALID_ARGUMENT;
  const bool dense = p->cu_seqlens_host == nullptr;
  for (const int64_t* s3 : {q_strides, k_strides, v_strides})
    for (int i = dense ? 0 : 1; i < 3; ++i)
      if (s3[i] < p->head_dim) return SAGE_ERR_INVALID_ARGUMENT;
  if (workspace_bytes < sz.workspace_qkv) return SAGE_ERR_INVALID_ARGUMENT;
  if ((st = device_ok(stream)) != SAGE_OK) return st;
  const int64_t ntok = dense ? p->seqlen : p->cu_seqlens_host[p->batch];
  FusedQuantArgs a{};
  CUtensorMap mq, mk, mv;
  int dt = 0, dh = 0, db = 0, dt2 = 0, dh2 = 0, db2 = 0, dt3 = 0, dh3 = 0, db3 = 0;
  if (!make_input_map(&mq, q, p, p->heads_q, q_strides, ntok, &dt, &dh, &db) ||
      !make_input_map(&mk, k, p, p->heads_kv, k_strides, ntok, &dt2, &dh2, &db2) ||
      !make_input_map(&mv, v, p, p->heads_kv, v_strides, ntok, &dt3, &dh3, &db3))
    return SAGE_ERR_CUDA;
  // the kernel addresses all three maps with one coordinate order
  if (dt != dt2 || dt != dt3 || dh != dh2 || dh != dh3 || db != db2 || db != db3)
    return SAGE_ERR_INVALID_ARGUMENT;
  a.dim_tok = dt; a.dim_head = dh; a.dim_batch = db;
  a.q8 = q8; a.q_scale = q_scale; a.k8 = k8; a.k_scale = k_scale; a.k_mean = k_mean;
  a.v8 = v8; a.v_scale = v_scale;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  a.ksum = reinterpret_cast<double*>(ws);
  ws += round_up(sz.workspace_qk, 256);
  a.vpart = reinterpret_cast<float*>(ws);
  ws += round_up(static_cast<size_t>(p->heads_kv) * (L.t_pad / kPad) * p->head_dim * sizeof(float), 256);
  a.vmax = reinterpret_cast<float*>(ws);
  a.hq = p->heads_q; a.hkv = p->heads_kv; a.nblk = static_cast<int>(L.t_pad / kPad);
  a.batch = p->batch;
  a.fine = p->granularity == SAGE_GRAN_THREAD ? 1 : 0;
  a.pv16 = p->pv == SAGE_PV_FP16 ? 1 : 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  return L.varlen ? dispatch_quant_fused(*L.var, p, mq, mk, mv, a, s)
                  : dispatch_quant_fused(L.dense, p, mq, mk, mv, a, s);
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
  if ((st = device_ok(stream)) != SAGE_OK) return st;
  const int d = p->head_dim;
  const uint64_t tp = static_cast<uint64_t>(L.t_pad);
  const bool pv16 = p->pv == SAGE_PV_FP16;
  const uint64_t vrow = tp * (pv16 ? 2 : 1);  // bytes per V^T row
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q8, d, tp * p->heads_q, d, d, kBlkQ, qk_swizzle(d)) ||
      !make_map(&mk, k8, d, tp * p->heads_kv, d, d, kKvTile, qk_swizzle(d)) ||
      !make_map(&mv, v8, vrow, static_cast<uint64_t>(p->heads_kv) * d, vrow, 128, d,
                CU_TENSOR_MAP_SWIZZLE_128B))
    return SAGE_ERR_CUDA;
  AttnArgs a{};
  a.q_scale = q_scale; a.k_scale = k_scale; a.v_scale = v_scale;
  a.out = out; a.out_dtype = static_cast<int>(out_dtype);
  a.osb = out_strides[0]; a.osh = out_strides[1]; a.ost = out_strides[2];
  a.lse = lse;
  a.hq = p->heads_q; a.hkv = p->heads_kv; a.group = p->heads_q / p->heads_kv;
  // fp64, as the definition forms the logits: 1/sqrt(d) unless the caller gives one
  a.scale = sm_scale > 0.0f ? static_cast<double>(sm_scale) : 1.0 / std::sqrt(static_cast<double>(d));
  a.causal = is_causal ? 1 : 0;
  const bool fine = p->granularity == SAGE_GRAN_THREAD;
  const int pv = !pv16 ? kPvE4m3 : (p->dtype == SAGE_BF16 ? kPvBf16 : kPvF16);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (L.varlen) {
    const int64_t ncta = L.var->cta[p->batch];
    if (ncta == 0) return SAGE_OK;
    return dispatch_attn(*L.var, ncta, d, fine, pv, mq, mk, mv, a, s);
  }
  const int64_t pairs = ((L.dense.len + kBlkQ - 1) / kBlkQ + 1) / 2;
  const int64_t ncta = static_cast<int64_t>(p->batch) * p->heads_q * pairs;
  return dispatch_attn(L.dense, ncta, d, fine, pv, mq, mk, mv, a, s);
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
  if ((st = device_ok(stream)) != SAGE_OK) return st;
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

sage_status_t sage_debug_watchdog_selftest(unsigned int limit_us, sage_stream_t stream) {
  if (limit_us == 0 || limit_us > 1000000u) return SAGE_ERR_INVALID_ARGUMENT;
  sage_status_t st = device_ok(stream);
  if (st != SAGE_OK) return st;
  watchdog_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<uint64_t>(limit_us) * 1000ull);
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
  if ((st = device_ok(stream)) != SAGE_OK) return st;
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

// ---------------------------------------------------------------------------
// sage_attn_host: the path on host buffers, pipelined over chunks of heads.
// ---------------------------------------------------------------------------
namespace {

// Per device: the copy-in and copy-out streams and the events that order a chunk's
// copy-in, kernels and copy-out across them (two workspace slots).
struct HostPipe {
  bool ready = false;
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t entry = nullptr, last = nullptr;
  cudaEvent_t in_done[2] = {nullptr, nullptr}, k_done[2] = {nullptr, nullptr},
              out_done[2] = {nullptr, nullptr};
};
std::mutex g_pipe_mu;
HostPipe g_pipe[kMaxDevices];

sage_status_t pipe_for_device(HostPipe** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SAGE_ERR_CUDA;
  HostPipe& P = g_pipe[dev];
  if (!P.ready) {
    const unsigned ef = cudaEventDisableTiming;
    bool ok = cudaStreamCreateWithFlags(&P.h2d, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&P.d2h, cudaStreamNonBlocking) == cudaSuccess &&
              cudaEventCreateWithFlags(&P.entry, ef) == cudaSuccess &&
              cudaEventCreateWithFlags(&P.last, ef) == cudaSuccess;
    for (int i = 0; i < 2 && ok; ++i)
      ok = cudaEventCreateWithFlags(&P.in_done[i], ef) == cudaSuccess &&
           cudaEventCreateWithFlags(&P.k_done[i], ef) == cudaSuccess &&
           cudaEventCreateWithFlags(&P.out_done[i], ef) == cudaSuccess;
    if (!ok) return SAGE_ERR_CUDA;
    P.ready = true;
  }
  *out = &P;
  return SAGE_OK;
}

size_t dtype_bytes(sage_dtype_t t) { return t == SAGE_FP32 ? 4 : 2; }
size_t up256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// The buffers of one workspace slot for a chunk problem of hc KV heads.
struct Slot {
  uint8_t *q, *k, *v, *out;
  int8_t *q8, *k8;
  float *q_scale, *k_scale, *k_mean, *v_scale;
  uint8_t* v8;
  void *ws_qk, *ws_v;
  size_t ws_qk_bytes, ws_v_bytes, bytes;
};

// Lay out one slot from `base` (or only measure it when base is null).
bool carve_slot(const sage_problem_t& cp, sage_dtype_t out_dtype, uint8_t* base, Slot* s) {
  sage_sizes_t sz;
  if (sage_buffer_sizes(&cp, &sz) != SAGE_OK) return false;
  const size_t hd = static_cast<size_t>(cp.seqlen) * cp.head_dim;
  const size_t in_q = static_cast<size_t>(cp.heads_q) * hd * 2, in_kv = static_cast<size_t>(cp.heads_kv) * hd * 2;
  const size_t o = static_cast<size_t>(cp.heads_q) * hd * dtype_bytes(out_dtype);
  size_t off = 0;
  auto take = [&](size_t n) { uint8_t* ptr = base ? base + off : nullptr; off += up256(n); return ptr; };
  s->q = take(in_q);
  s->k = take(in_kv);
  s->v = take(in_kv);
  s->out = take(o);
  s->q8 = reinterpret_cast<int8_t*>(take(sz.q8));
  s->q_scale = reinterpret_cast<float*>(take(sz.q_scale));
  s->k8 = reinterpret_cast<int8_t*>(take(sz.k8));
  s->k_scale = reinterpret_cast<float*>(take(sz.k_scale));
  s->k_mean = reinterpret_cast<float*>(take(sz.k_mean));
  s->v8 = take(sz.v8);
  s->v_scale = reinterpret_cast<float*>(take(sz.v_scale));
  s->ws_qk = take(sz.workspace_qk);
  s->ws_v = take(sz.workspace_v);
  s->ws_qk_bytes = sz.workspace_qk;
  s->ws_v_bytes = sz.workspace_v;
  s->bytes = off;
  return true;
}

int chunk_heads(const sage_problem_t* p, int kv_heads_per_chunk) {
  int hc = kv_heads_per_chunk;
  if (hc <= 0) {  // at least 8 chunks over the whole problem where the heads allow it
    const int64_t units = static_cast<int64_t>(p->batch) * p->heads_kv;
    hc = static_cast<int>(units / 8 < 1 ? 1 : units / 8);
  }
  return hc < p->heads_kv ? hc : p->heads_kv;
}

sage_problem_t chunk_problem(const sage_problem_t* p, int hc) {
  sage_problem_t cp = *p;
  const int g = p->heads_q / p->heads_kv;
  cp.batch = 1;
  cp.heads_kv = hc;
  cp.heads_q = hc * g;
  cp.cu_seqlens_host = nullptr;
  return cp;
}

}  // namespace

extern "C" size_t sage_host_workspace_bytes(const sage_problem_t* p, int kv_heads_per_chunk,
                                            sage_dtype_t out_dtype) {
  Layout L;
  if (p == nullptr || p->cu_seqlens_host != nullptr || plan(p, L, nullptr) != SAGE_OK) return 0;
  const sage_problem_t cp = chunk_problem(p, chunk_heads(p, kv_heads_per_chunk));
  Slot s;
  if (!carve_slot(cp, out_dtype, nullptr, &s)) return 0;
  return 2 * s.bytes;
}

extern "C" sage_status_t sage_attn_host(const sage_problem_t* p, int tensor_layout,
                                        const void* q_host, const void* k_host, const void* v_host,
                                        void* out_host, sage_dtype_t out_dtype, float sm_scale,
                                        int is_causal, int kv_heads_per_chunk, void* workspace,
                                        size_t workspace_bytes, sage_stream_t stream) {
  Layout L;
  if (p == nullptr || p->cu_seqlens_host != nullptr) return SAGE_ERR_INVALID_ARGUMENT;
  sage_status_t st = plan(p, L, nullptr);
  if (st != SAGE_OK) return st;
  if (tensor_layout != 0 && tensor_layout != 1) return SAGE_ERR_INVALID_ARGUMENT;
  if (out_dtype != SAGE_FP16 && out_dtype != SAGE_BF16 && out_dtype != SAGE_FP32)
    return SAGE_ERR_INVALID_ARGUMENT;
  if (!q_host || !k_host || !v_host || !out_host || !workspace) return SAGE_ERR_INVALID_ARGUMENT;
  if (!aligned16(q_host) || !aligned16(k_host) || !aligned16(v_host) || !aligned16(out_host) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return SAGE_ERR_INVALID_ARGUMENT;
  const int hc = chunk_heads(p, kv_heads_per_chunk);
  const sage_problem_t cfull = chunk_problem(p, hc);
  Slot slot[2];
  if (!carve_slot(cfull, out_dtype, nullptr, &slot[0])) return SAGE_ERR_INVALID_ARGUMENT;
  // every slot is as large as a full chunk needs; a short last chunk must not move
  // the base of the next slot
  const size_t slot_bytes = slot[0].bytes;
  if (workspace_bytes < 2 * slot_bytes) return SAGE_ERR_INVALID_ARGUMENT;
  if ((st = device_ok(stream)) != SAGE_OK) return st;

  std::lock_guard<std::mutex> lock(g_pipe_mu);
  HostPipe* P = nullptr;
  if ((st = pipe_for_device(&P)) != SAGE_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int g = p->heads_q / p->heads_kv;
  const int64_t N = p->seqlen, d = p->head_dim;
  const size_t ib = 2, ob = dtype_bytes(out_dtype);
  // element strides {batch, head, token} of a chunk in its slot
  auto slot_strides = [&](int heads, int64_t (&st3)[3]) {
    if (tensor_layout == 0) { st3[0] = heads * N * d; st3[1] = N * d; st3[2] = d; }
    else { st3[0] = N * heads * d; st3[1] = d; st3[2] = heads * d; }
  };
  // copy `heads` heads starting at head h0 of batch entry b between a host array of
  // H heads and a contiguous slot buffer holding just those heads
  auto copy = [&](void* dst, const void* src, int b, int h0, int heads, int H, size_t eb, bool to_dev,
                  cudaStream_t cs) -> bool {
    const size_t row = static_cast<size_t>(d) * eb;  // one (token, head) row
    if (tensor_layout == 0) {
      const size_t host_off = (static_cast<size_t>(b) * H + h0) * N * row;
      const size_t n = static_cast<size_t>(heads) * N * row;
      return to_dev ? cudaMemcpyAsync(dst, static_cast<const uint8_t*>(src) + host_off, n,
                                      cudaMemcpyHostToDevice, cs) == cudaSuccess
                    : cudaMemcpyAsync(static_cast<uint8_t*>(dst) + host_off, src, n,
                                      cudaMemcpyDeviceToHost, cs) == cudaSuccess;
    }
    const size_t host_off = static_cast<size_t>(b) * N * H * row + h0 * row;
    const size_t hpitch = H * row, dpitch = heads * row, width = heads * row;
    return to_dev ? cudaMemcpy2DAsync(dst, dpitch, static_cast<const uint8_t*>(src) + host_off, hpitch,
                                      width, N, cudaMemcpyHostToDevice, cs) == cudaSuccess
                  : cudaMemcpy2DAsync(static_cast<uint8_t*>(dst) + host_off, hpitch, src, dpitch,
                                      width, N, cudaMemcpyDeviceToHost, cs) == cudaSuccess;
  };

  // the slots' previous users are the work already enqueued on `stream`
  if (cudaEventRecord(P->entry, s) != cudaSuccess ||
      cudaStreamWaitEvent(P->h2d, P->entry, 0) != cudaSuccess)
    return SAGE_ERR_CUDA;
  int c = 0;
  for (int b = 0; b < p->batch; ++b) {
    for (int h0 = 0; h0 < p->heads_kv; h0 += hc, ++c) {
      const int heads = (p->heads_kv - h0 < hc) ? p->heads_kv - h0 : hc;
      const sage_problem_t cp = chunk_problem(p, heads);
      const int i = c & 1;
      carve_slot(cp, out_dtype, static_cast<uint8_t*>(workspace) + i * slot_bytes, &slot[i]);
      Slot& S = slot[i];
      // copy-in: the slot's inputs are free once chunk c-2's kernels are done
      if (c >= 2 && cudaStreamWaitEvent(P->h2d, P->k_done[i], 0) != cudaSuccess) return SAGE_ERR_CUDA;
      if (!copy(S.q, q_host, b, h0 * g, heads * g, p->heads_q, ib, true, P->h2d) ||
          !copy(S.k, k_host, b, h0, heads, p->heads_kv, ib, true, P->h2d) ||
          !copy(S.v, v_host, b, h0, heads, p->heads_kv, ib, true, P->h2d) ||
          cudaEventRecord(P->in_done[i], P->h2d) != cudaSuccess)
        return SAGE_ERR_CUDA;
      // kernels on `stream`: after the copy-in, and after chunk c-2's copy-out has
      // read this slot's output buffer
      if (cudaStreamWaitEvent(s, P->in_done[i], 0) != cudaSuccess) return SAGE_ERR_CUDA;
      if (c >= 2 && cudaStreamWaitEvent(s, P->out_done[i], 0) != cudaSuccess) return SAGE_ERR_CUDA;
      int64_t qs[3], ks[3];
      slot_strides(heads * g, qs);
      slot_strides(heads, ks);
      if ((st = sage_quant_qk(&cp, S.q, qs, S.k, ks, S.q8, S.q_scale, S.k8, S.k_scale, S.k_mean,
                              S.ws_qk, S.ws_qk_bytes, stream)) != SAGE_OK)
        return st;
      if ((st = sage_quant_v(&cp, S.v, ks, S.v8, S.v_scale, S.ws_v, S.ws_v_bytes, stream)) != SAGE_OK)
        return st;
      if ((st = sage_attn_fwd(&cp, S.q8, S.q_scale, S.k8, S.k_scale, S.v8, S.v_scale, sm_scale,
                              is_causal, S.out, out_dtype, qs, nullptr, stream)) != SAGE_OK)
        return st;
      if (cudaEventRecord(P->k_done[i], s) != cudaSuccess) return SAGE_ERR_CUDA;
      // copy-out
      if (cudaStreamWaitEvent(P->d2h, P->k_done[i], 0) != cudaSuccess ||
          !copy(out_host, S.out, b, h0 * g, heads * g, p->heads_q, ob, false, P->d2h) ||
          cudaEventRecord(P->out_done[i], P->d2h) != cudaSuccess)
        return SAGE_ERR_CUDA;
    }
  }
  // `stream` continues after the last copy-out
  if (cudaEventRecord(P->last, P->d2h) != cudaSuccess || cudaStreamWaitEvent(s, P->last, 0) != cudaSuccess)
    return SAGE_ERR_CUDA;
  return SAGE_OK;
}

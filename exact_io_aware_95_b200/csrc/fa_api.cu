// C-ABI entry points of the exact-attention library (declared in include/fa.h):
// host-side validation, TMA tensor-map construction, template dispatch and
// launch.  No device memory is allocated here; no compute happens on the host.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "fa.h"

#include "fa_bwd.cuh"
#include "fa_bwd_dq.cuh"
#include "fa_decode.cuh"
#include "fa_fwd.cuh"
#include "fa_fwd_fp8.cuh"

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

std::mutex g_mu;

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!tried) {
    tried = true;
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

CtxGetCurrentFn ctx_get_current_fn() {
  static CtxGetCurrentFn fn = nullptr;
  static bool tried = false;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!tried) {
    tried = true;
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(ptr);
  }
  return fn;
}

// A host thread that has not yet made any CUDA context current (a new worker
// thread, e.g. the one torch's autograd engine runs a backward on) gets one
// lazily from the first runtime call that needs it; the driver's tensor-map
// encoder, called before any such runtime call, would fail with
// CUDA_ERROR_INVALID_CONTEXT.  Bind the current device's primary context in
// that case.  A context the caller made current is left untouched.
bool bind_context_if_none(int dev) {
  CtxGetCurrentFn get = ctx_get_current_fn();
  CUcontext ctx = nullptr;
  if (get && get(&ctx) == CUDA_SUCCESS && ctx != nullptr) return true;
  if (cudaSetDevice(dev) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return true;
}

constexpr int kMaxDevices = 64;

// Per-device: compute capability check result and the opt-in shared-memory
// attribute of each kernel instantiation (set once per device).
struct DeviceState {
  int checked = 0;  // 0 unknown, 1 sm_100, -1 other
};
DeviceState g_dev[kMaxDevices];

fa_status current_device(int* dev) {
  if (cudaGetDevice(dev) != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_CUDA;
  }
  if (*dev < 0 || *dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
  if (!bind_context_if_none(*dev)) return FA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState& st = g_dev[*dev];
  if (st.checked == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, *dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, *dev) != cudaSuccess) {
      cudaGetLastError();
      return FA_ERR_CUDA;
    }
    st.checked = (major == 10 && minor == 0) ? 1 : -1;
  }
  return st.checked == 1 ? FA_OK : FA_ERR_UNSUPPORTED;
}

// Set the dynamic shared-memory limit of `kern` once per device.  Kernels
// that re-balance registers between warpgroups (setmaxnreg) must have been
// compiled to exactly the register count their split was planned for (the
// split adds up to the launch allocation; a larger one would never be
// granted).  Refuse to launch such a kernel otherwise.
template <typename K>
fa_status ensure_smem(K kern, int dev, int bytes, bool* done_flags, int need_regs = 0) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!done_flags[dev]) {
    if (need_regs) {
      cudaFuncAttributes attr;
      if (cudaFuncGetAttributes(&attr, kern) != cudaSuccess) {
        cudaGetLastError();
        return FA_ERR_CUDA;
      }
      if (attr.numRegs != need_regs) return FA_ERR_UNSUPPORTED;
    }
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) {
      cudaGetLastError();
      return FA_ERR_CUDA;
    }
    done_flags[dev] = true;
  }
  return FA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Tensor map over a bf16 array laid out [outer, rows, H, d] (d innermost),
// read in boxes of 64 (d) x 1 (head) x box_rows (rows) with 128-byte swizzle.
fa_status make_map_bf16(CUtensorMap* m, const void* base, int d, int H, int64_t rows, int64_t outer,
                        int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return FA_ERR_CUDA;
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)rows, (cuuint64_t)outer};
  cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2, (cuuint64_t)rows * H * d * 2};
  cuuint32_t box[4] = {64, 1, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

// Tensor map over a byte array (e4m3) with dims {d0, d1, d2, d3} (d0
// innermost, contiguous), row pitches in bytes, boxes {b0, b1, b2, 1} and
// 128-byte swizzle.
fa_status make_map_u8(CUtensorMap* m, const void* base, const uint64_t (&dims)[4], const uint64_t (&pitch)[3],
                      const uint32_t (&box)[3]) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return FA_ERR_CUDA;
  cuuint64_t gd[4] = {dims[0], dims[1], dims[2], dims[3]};
  cuuint64_t gs[3] = {pitch[0], pitch[1], pitch[2]};
  cuuint32_t bx[4] = {box[0], box[1], box[2], 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(base), gd, gs, bx, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

// Measurement hook (fa_record_launch_events): caller-created CUDA events that
// the next compute call of this host thread records between its launches.
struct LaunchEvents {
  cudaEvent_t ev[8];
  int n = 0;
  int used = 0;
};
thread_local LaunchEvents t_launch_events;

void mark_launch(cudaStream_t s) {
  LaunchEvents& h = t_launch_events;
  if (h.used < h.n && cudaEventRecord(h.ev[h.used], s) == cudaSuccess) ++h.used;
}

// Clears the hook when a public compute call returns, however it returns.
struct LaunchEventsScope {
  ~LaunchEventsScope() { t_launch_events.n = t_launch_events.used = 0; }
};

fa_status launch_status(cudaStream_t s) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return FA_ERR_CUDA;
  mark_launch(s);
  return FA_OK;
}

constexpr float kLog2e = 1.4426950408889634f;

// Heads per scheduling group: as many as keep `bytes_per_head` of streamed
// operands within a share of the 126 MB L2, at least 1, at most all heads.
int head_group(int64_t bytes_per_head, int64_t heads) {
  constexpr int64_t kL2Budget = 48ll << 20;
  int64_t g = bytes_per_head > 0 ? kL2Budget / bytes_per_head : heads;
  if (g < 1) g = 1;
  if (g > heads) g = heads;
  return static_cast<int>(g);
}

// ------------------------------------------------------------------ forward
template <int D, bool CAUSAL, bool VARLEN>
fa_status launch_fwd(int dev, const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                     const fa::FwdParams& p, cudaStream_t s) {
  static bool done[kMaxDevices] = {};
  auto kern = fa::fa_fwd_kernel<D, CAUSAL, VARLEN>;
  constexpr int smem = fa::FwdCfg<D>::SMEM_BYTES;
  fa_status st = ensure_smem(kern, dev, smem, done, fa::kLaunchRegs);
  if (st != FA_OK) return st;
  // one CTA per work item; running CTAs take over the items of CTAs that have
  // not started (cluster launch control), so about one CTA per SM runs
  const int64_t grid = static_cast<int64_t>(p.npairs) * p.B * p.H;
  if (grid <= 0 || grid > 0x7fffffff) return FA_ERR_INVALID_ARG;
  mark_launch(s);
  kern<<<static_cast<unsigned>(grid), fa::FwdCfg<D>::THREADS, smem, s>>>(q, k, v, p);
  return launch_status(s);
}

template <int D>
fa_status dispatch_fwd(int dev, bool causal, bool varlen, const CUtensorMap& q, const CUtensorMap& k,
                       const CUtensorMap& v, const fa::FwdParams& p, cudaStream_t s) {
  if (varlen) return causal ? launch_fwd<D, true, true>(dev, q, k, v, p, s) : launch_fwd<D, false, true>(dev, q, k, v, p, s);
  return causal ? launch_fwd<D, true, false>(dev, q, k, v, p, s) : launch_fwd<D, false, false>(dev, q, k, v, p, s);
}

fa_status fwd_common(const void* q, const void* k, const void* v, void* o, float* lse, const int* cu, int B,
                     int N, int total, int H, int d, float scale, int causal, void* stream) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return FA_ERR_INVALID_ARG;
  if (B < 1 || N < 1 || H < 1 || total < 1) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  const bool varlen = cu != nullptr;
  const int64_t rows = varlen ? total : N;
  const int64_t outer = varlen ? 1 : B;
  if (rows * outer * H * d > (int64_t(1) << 40)) return FA_ERR_INVALID_ARG;
  int dev;
  fa_status st = current_device(&dev);
  if (st != FA_OK) return st;
  CUtensorMap mq, mk, mv;
  if ((st = make_map_bf16(&mq, q, d, H, rows, outer, 128)) != FA_OK) return st;
  if ((st = make_map_bf16(&mk, k, d, H, rows, outer, 128)) != FA_OK) return st;
  if ((st = make_map_bf16(&mv, v, d, H, rows, outer, 128)) != FA_OK) return st;
  fa::FwdParams p;
  p.o = o;
  p.lse = lse;
  p.cu_seqlens = cu;
  p.B = B;
  p.N = N;
  p.H = H;
  p.total = varlen ? total : N;
  p.npairs = (N + 255) / 256;
  p.group = head_group(static_cast<int64_t>(N) * d * 2 * 2, static_cast<int64_t>(B) * H);  // K and V of one head
  p.scale_log2 = scale * kLog2e;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  return d == 64 ? dispatch_fwd<64>(dev, causal, varlen, mq, mk, mv, p, s)
                 : dispatch_fwd<128>(dev, causal, varlen, mq, mk, mv, p, s);
}

// ----------------------------------------------------------------- backward
// Grid of the memory-bound preprocess: grid-stride loops over a resident wave
// (8 blocks of 256 threads per SM).
unsigned preprocess_blocks(int dev) {
  int sms = 148;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    sms = 148;
  }
  return static_cast<unsigned>(sms * 8);
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

size_t ws_bytes_for(int64_t rows, int H, int d) {
  return align256(static_cast<size_t>(rows) * H * d * sizeof(float)) + align256(static_cast<size_t>(rows) * H * sizeof(float));
}

// Deterministic order: preprocess (D only), dK/dV kernel without its dQ
// product, then the dQ pass (fixed summation order, no atomics).
template <int D, bool CAUSAL, bool VARLEN>
fa_status launch_bwd_det(int dev, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                         const CUtensorMap& mdo, fa::BwdParams p, int dq_group, cudaStream_t s) {
  static bool done_main[kMaxDevices] = {};
  static bool done_dq[kMaxDevices] = {};
  auto kmain = fa::fa_bwd_kernel<D, CAUSAL, VARLEN, false>;
  auto kdq = fa::fa_bwd_dq_kernel<D, CAUSAL, VARLEN>;
  constexpr int smem_main = fa::BwdCfg<D>::SMEM_BYTES;
  constexpr int smem_dq = fa::DqCfg<D>::SMEM_BYTES;
  fa_status st = ensure_smem(kmain, dev, smem_main, done_main, fa::BwdCfg<D>::LAUNCH_REGS);
  if (st != FA_OK) return st;
  if ((st = ensure_smem(kdq, dev, smem_dq, done_dq)) != FA_OK) return st;
  p.dq_acc = nullptr;  // no accumulator: the preprocess computes D only
  const int64_t grid = static_cast<int64_t>(p.nkvtiles) * p.B * p.H;
  if (grid > 0x7fffffff) return FA_ERR_INVALID_ARG;
  {
    mark_launch(s);
    fa::fa_bwd_preprocess_kernel<D><<<preprocess_blocks(dev), 256, 0, s>>>(p);
    if ((st = launch_status(s)) != FA_OK) return st;
  }
  kmain<<<static_cast<unsigned>(grid), fa::BwdCfg<D>::THREADS, smem_main, s>>>(mq, mk, mv, mdo, p);
  if ((st = launch_status(s)) != FA_OK) return st;
  p.group = dq_group;
  kdq<<<static_cast<unsigned>(grid), fa::DqCfg<D>::THREADS, smem_dq, s>>>(mq, mk, mv, mdo, p);
  return launch_status(s);
}

template <int D, bool CAUSAL, bool VARLEN>
fa_status launch_bwd(int dev, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                     const CUtensorMap& mdo, const fa::BwdParams& p, cudaStream_t s) {
  static bool done[kMaxDevices] = {};
  auto kern = fa::fa_bwd_kernel<D, CAUSAL, VARLEN, true>;
  constexpr int smem = fa::BwdCfg<D>::SMEM_BYTES;
  fa_status st = ensure_smem(kern, dev, smem, done, fa::BwdCfg<D>::LAUNCH_REGS);
  if (st != FA_OK) return st;
  // 1) D = rowsum(dO * O) and zeroed dQ accumulator
  {
    mark_launch(s);
    fa::fa_bwd_preprocess_kernel<D><<<preprocess_blocks(dev), 256, 0, s>>>(p);
    if ((st = launch_status(s)) != FA_OK) return st;
  }
  // 2) fused recompute + dK, dV, dQ accumulation: one work item per 128-key tile, taken by persistent CTAs
  {
    const int64_t grid = static_cast<int64_t>(p.nkvtiles) * p.B * p.H;
    if (grid > 0x7fffffff) return FA_ERR_INVALID_ARG;
    kern<<<static_cast<unsigned>(grid), fa::BwdCfg<D>::THREADS, smem, s>>>(mq, mk, mv, mdo, p);
    if ((st = launch_status(s)) != FA_OK) return st;
  }
  // 3) dQ = bf16(scale * dQ accumulator)
  {
    const int64_t R = p.cu_seqlens ? p.total : p.N;
    const int64_t nbh = p.cu_seqlens ? p.H : static_cast<int64_t>(p.B) * p.H;
    const int64_t blocks = nbh * ((R + 31) / 32);
    if (blocks > 0x7fffffff) return FA_ERR_INVALID_ARG;
    fa::fa_bwd_dq_convert_kernel<D><<<static_cast<unsigned>(blocks), 256, 0, s>>>(p);
    if ((st = launch_status(s)) != FA_OK) return st;
  }
  return FA_OK;
}

template <int D>
fa_status dispatch_bwd(int dev, bool causal, bool varlen, const CUtensorMap& q, const CUtensorMap& k,
                       const CUtensorMap& v, const CUtensorMap& d_o, const fa::BwdParams& p, int dq_group,
                       bool det, cudaStream_t s) {
  if (det) {
    if (varlen)
      return causal ? launch_bwd_det<D, true, true>(dev, q, k, v, d_o, p, dq_group, s)
                    : launch_bwd_det<D, false, true>(dev, q, k, v, d_o, p, dq_group, s);
    return causal ? launch_bwd_det<D, true, false>(dev, q, k, v, d_o, p, dq_group, s)
                  : launch_bwd_det<D, false, false>(dev, q, k, v, d_o, p, dq_group, s);
  }
  if (varlen)
    return causal ? launch_bwd<D, true, true>(dev, q, k, v, d_o, p, s) : launch_bwd<D, false, true>(dev, q, k, v, d_o, p, s);
  return causal ? launch_bwd<D, true, false>(dev, q, k, v, d_o, p, s) : launch_bwd<D, false, false>(dev, q, k, v, d_o, p, s);
}

fa_status bwd_common(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                     void* dq, void* dk, void* dv, void* ws, size_t ws_bytes, const int* cu, int B, int N, int total,
                     int H, int d, float scale, int causal, void* stream, bool det = false) {
  if (!q || !k || !v || !o || !lse || !dO || !dq || !dk || !dv || !ws) return FA_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, o, lse, dO, dq, dk, dv, ws};
  for (const void* ptr : ptrs)
    if (!aligned16(ptr)) return FA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return FA_ERR_INVALID_ARG;
  if (B < 1 || N < 1 || H < 1 || total < 1) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  const bool varlen = cu != nullptr;
  const int64_t rows = varlen ? total : N;
  const int64_t outer = varlen ? 1 : B;
  if (rows * outer * H * d > (int64_t(1) << 40)) return FA_ERR_INVALID_ARG;
  const size_t need = ws_bytes_for(rows * outer, H, d);
  if (ws_bytes < need) return FA_ERR_WORKSPACE;
  int dev;
  fa_status st = current_device(&dev);
  if (st != FA_OK) return st;
  CUtensorMap mq, mk, mv, mdo;
  if ((st = make_map_bf16(&mq, q, d, H, rows, outer, 128)) != FA_OK) return st;
  if ((st = make_map_bf16(&mk, k, d, H, rows, outer, 128)) != FA_OK) return st;
  if ((st = make_map_bf16(&mv, v, d, H, rows, outer, 128)) != FA_OK) return st;
  if ((st = make_map_bf16(&mdo, dO, d, H, rows, outer, 128)) != FA_OK) return st;
  fa::BwdParams p;
  p.o = o;
  p.dout = dO;
  p.lse = lse;
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  p.dq_acc = static_cast<float*>(ws);
  p.dvec = reinterpret_cast<float*>(static_cast<char*>(ws) + align256(static_cast<size_t>(rows * outer) * H * d * sizeof(float)));
  p.cu_seqlens = cu;
  p.B = B;
  p.N = N;
  p.H = H;
  p.total = varlen ? total : N;
  p.rows = static_cast<int>(rows * outer);
  p.nkvtiles = (N + 127) / 128;
  p.group = head_group(static_cast<int64_t>(N) * d * (2 + 2 + 4), static_cast<int64_t>(B) * H);  // Q, dO, dQ acc
  p.scale = scale;
  p.scale_log2 = scale * kLog2e;
  // the dQ pass streams K and V of a head once per query tile
  const int dq_group = head_group(static_cast<int64_t>(N) * d * 2 * 2, static_cast<int64_t>(B) * H);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  return d == 64 ? dispatch_bwd<64>(dev, causal, varlen, mq, mk, mv, mdo, p, dq_group, det, s)
                 : dispatch_bwd<128>(dev, causal, varlen, mq, mk, mv, mdo, p, dq_group, det, s);
}

// ----------------------------------------------------------------- decode
// Workspace: prefix [B + 1] int64 | bad-length flag | records rec_o
// [G][2][Nq][d] fp32 | rec_lse [G][2][Nq] fp32, each part 256-byte aligned.
// It depends on B, Nq and d only.
struct DecodeWs {
  size_t prefix, bad, rec_o, rec_lse, total;
};
DecodeWs decode_ws_layout(int B, int Nq, int d) {
  DecodeWs w;
  const size_t recs = static_cast<size_t>(fa::kDecodeGrid) * 2 * Nq;
  w.prefix = 0;
  w.bad = align256((static_cast<size_t>(B) + 1) * sizeof(long long));
  w.rec_o = w.bad + 256;
  w.rec_lse = w.rec_o + align256(recs * d * sizeof(float));
  w.total = w.rec_lse + align256(recs * sizeof(float));
  return w;
}

template <int D, int NQ>
fa_status launch_decode(int dev, const CUtensorMap& mk, const CUtensorMap& mv, const fa::DecParams& p,
                        cudaStream_t s) {
  static bool done[kMaxDevices] = {};
  auto kern = fa::fa_decode_stream_kernel<D, NQ>;
  constexpr int smem = fa::DecCfg<D, NQ>::SMEM_BYTES;
  fa_status st = ensure_smem(kern, dev, smem, done);
  if (st != FA_OK) return st;
  mark_launch(s);
  fa::fa_decode_prefix_kernel<<<1, 256, 0, s>>>(p);
  if ((st = launch_status(s)) != FA_OK) return st;
  kern<<<static_cast<unsigned>(p.grid), fa::DecCfg<D, NQ>::THREADS, smem, s>>>(mk, mv, p);
  if ((st = launch_status(s)) != FA_OK) return st;
  const int64_t rows = static_cast<int64_t>(p.B) * p.H * p.Nq;
  fa::fa_decode_merge_kernel_impl<<<static_cast<unsigned>((rows + 3) / 4), 128, 4 * p.grid * sizeof(float), s>>>(p, D);
  return launch_status(s);
}

bool valid_cu(const int* cu, int nseq, int total, int max_seqlen) {
  return cu && nseq >= 1 && total >= 1 && max_seqlen >= 1;
}

}  // namespace

extern "C" {

fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int N, int H, int d,
                 float scale, int causal, void* stream) {
  LaunchEventsScope hook_scope;
  return fwd_common(q, k, v, o, lse, nullptr, B, N, N, H, d, scale, causal, stream);
}

fa_status fa_varlen_fwd(const void* q, const void* k, const void* v, void* o, float* lse, const int* cu_seqlens,
                        int nseq, int total, int max_seqlen, int H, int d, float scale, int causal, void* stream) {
  LaunchEventsScope hook_scope;
  if (!valid_cu(cu_seqlens, nseq, total, max_seqlen)) return FA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) != 0) return FA_ERR_INVALID_ARG;
  return fwd_common(q, k, v, o, lse, cu_seqlens, nseq, max_seqlen, total, H, d, scale, causal, stream);
}

size_t fa_bwd_workspace_size(int B, int N, int H, int d) {
  if (B < 1 || N < 1 || H < 1 || (d != 64 && d != 128)) return 0;
  return ws_bytes_for(static_cast<int64_t>(B) * N, H, d);
}

fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                 void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes, int B, int N, int H, int d,
                 float scale, int causal, void* stream) {
  LaunchEventsScope hook_scope;
  return bwd_common(q, k, v, o, lse, dO, dq, dk, dv, workspace, ws_bytes, nullptr, B, N, N, H, d, scale, causal,
                    stream);
}

fa_status fa_varlen_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                        void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes, const int* cu_seqlens,
                        int nseq, int total, int max_seqlen, int H, int d, float scale, int causal, void* stream) {
  LaunchEventsScope hook_scope;
  if (!valid_cu(cu_seqlens, nseq, total, max_seqlen)) return FA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) != 0) return FA_ERR_INVALID_ARG;
  return bwd_common(q, k, v, o, lse, dO, dq, dk, dv, workspace, ws_bytes, cu_seqlens, nseq, max_seqlen, total, H, d,
                    scale, causal, stream);
}

fa_status fa_bwd_deterministic(const void* q, const void* k, const void* v, const void* o, const float* lse,
                               const void* dO, void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes, int B,
                               int N, int H, int d, float scale, int causal, void* stream) {
  LaunchEventsScope hook_scope;
  return bwd_common(q, k, v, o, lse, dO, dq, dk, dv, workspace, ws_bytes, nullptr, B, N, N, H, d, scale, causal,
                    stream, true);
}

fa_status fa_varlen_bwd_deterministic(const void* q, const void* k, const void* v, const void* o, const float* lse,
                                      const void* dO, void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes,
                                      const int* cu_seqlens, int nseq, int total, int max_seqlen, int H, int d,
                                      float scale, int causal, void* stream) {
  LaunchEventsScope hook_scope;
  if (!valid_cu(cu_seqlens, nseq, total, max_seqlen)) return FA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(cu_seqlens) & 3u) != 0) return FA_ERR_INVALID_ARG;
  return bwd_common(q, k, v, o, lse, dO, dq, dk, dv, workspace, ws_bytes, cu_seqlens, nseq, max_seqlen, total, H, d,
                    scale, causal, stream, true);
}

size_t fa_decode_workspace_size(int B, int Nq, int Nk, int H, int d) {
  if (B < 1 || Nq < 1 || Nq > 16 || Nk < 1 || H < 1 || (d != 64 && d != 128)) return 0;
  return decode_ws_layout(B, Nq, d).total;
}

fa_status fa_decode_fwd(const void* q, const void* k_cache, const void* v_cache, void* o, float* lse,
                        const int* seqlens_k, void* workspace, size_t ws_bytes, int B, int Nq, int Nk, int H, int d,
                        float scale, int causal, void* stream) {
  LaunchEventsScope hook_scope;
  if (!q || !k_cache || !v_cache || !o || !lse) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o) || !aligned16(lse))
    return FA_ERR_INVALID_ARG;
  if (seqlens_k && (reinterpret_cast<uintptr_t>(seqlens_k) & 3u) != 0) return FA_ERR_INVALID_ARG;
  if (B < 1 || Nq < 1 || Nk < 1 || H < 1) return FA_ERR_INVALID_ARG;
  if (Nq > 16) return FA_ERR_UNSUPPORTED;
  if (B > 65535 || H > 65535) return FA_ERR_INVALID_ARG;  // grid y / z limits
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(B) * Nk * H * d > (int64_t(1) << 40)) return FA_ERR_INVALID_ARG;
  const DecodeWs wl = decode_ws_layout(B, Nq, d);
  if (!workspace || ws_bytes < wl.total) return FA_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return FA_ERR_INVALID_ARG;
  int dev;
  fa_status st = current_device(&dev);
  if (st != FA_OK) return st;
  CUtensorMap mk, mv;
  if ((st = make_map_bf16(&mk, k_cache, d, H, Nk, B, 64)) != FA_OK) return st;  // 64-key tiles
  if ((st = make_map_bf16(&mv, v_cache, d, H, Nk, B, 64)) != FA_OK) return st;
  fa::DecParams p;
  p.q = q;
  p.o = o;
  p.lse = lse;
  p.seqlens = seqlens_k;
  p.B = B;
  p.Nq = Nq;
  p.Nk = Nk;
  p.H = H;
  char* ws = static_cast<char*>(workspace);
  p.prefix = reinterpret_cast<long long*>(ws + wl.prefix);
  p.bad = reinterpret_cast<int*>(ws + wl.bad);
  p.rec_o = reinterpret_cast<float*>(ws + wl.rec_o);
  p.rec_lse = reinterpret_cast<float*>(ws + wl.rec_lse);
  p.grid = fa::kDecodeGrid;
  p.causal = causal;
  p.scale_log2 = scale * kLog2e;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (d == 64) return Nq == 1 ? launch_decode<64, 1>(dev, mk, mv, p, s) : launch_decode<64, 16>(dev, mk, mv, p, s);
  return Nq == 1 ? launch_decode<128, 1>(dev, mk, mv, p, s) : launch_decode<128, 16>(dev, mk, mv, p, s);
}

size_t fa_fwd_fp8_workspace_size(int B, int N, int H, int d) {
  if (B < 1 || N < 1 || H < 1 || d != 128) return 0;
  const size_t npad = (static_cast<size_t>(N) + 15) / 16 * 16;
  return align256(static_cast<size_t>(B) * H * 128 * npad);
}

fa_status fa_fwd_fp8(const void* q, const void* k, const void* v, float descale_q, float descale_k, float descale_v,
                     void* o, float* lse, void* workspace, size_t ws_bytes, int B, int N, int H, int d, float scale,
                     int causal, void* stream) {
  LaunchEventsScope hook_scope;
  if (!q || !k || !v || !o || !lse || !workspace) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return FA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return FA_ERR_INVALID_ARG;
  if (B < 1 || N < 1 || H < 1) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (!std::isfinite(scale) || !std::isfinite(descale_q) || !std::isfinite(descale_k) || !std::isfinite(descale_v) ||
      !(descale_q > 0.f) || !(descale_k > 0.f) || !(descale_v > 0.f))
    return FA_ERR_INVALID_ARG;
  if (d != 128) return FA_ERR_UNSUPPORTED;
  if (B > 65535 || H > 65535) return FA_ERR_INVALID_ARG;  // transpose grid y / z
  if (static_cast<int64_t>(B) * N * H * d > (int64_t(1) << 40)) return FA_ERR_INVALID_ARG;
  if (ws_bytes < fa_fwd_fp8_workspace_size(B, N, H, d)) return FA_ERR_WORKSPACE;
  int dev;
  fa_status st = current_device(&dev);
  if (st != FA_OK) return st;
  const uint64_t npad = (static_cast<uint64_t>(N) + 15) / 16 * 16;
  CUtensorMap mq, mk, mvt;
  {
    const uint64_t dims[4] = {128, static_cast<uint64_t>(H), static_cast<uint64_t>(N), static_cast<uint64_t>(B)};
    const uint64_t pitch[3] = {128, static_cast<uint64_t>(H) * 128, static_cast<uint64_t>(N) * H * 128};
    const uint32_t box[3] = {128, 1, 128};
    if ((st = make_map_u8(&mq, q, dims, pitch, box)) != FA_OK) return st;
    if ((st = make_map_u8(&mk, k, dims, pitch, box)) != FA_OK) return st;
  }
  {
    const uint64_t dims[4] = {npad, 128, static_cast<uint64_t>(H), static_cast<uint64_t>(B)};
    const uint64_t pitch[3] = {npad, 128 * npad, static_cast<uint64_t>(H) * 128 * npad};
    const uint32_t box[3] = {128, 128, 1};
    if ((st = make_map_u8(&mvt, workspace, dims, pitch, box)) != FA_OK) return st;
  }
  static bool done_nc[kMaxDevices] = {}, done_c[kMaxDevices] = {};
  auto kern = causal ? fa::fa_fwd_fp8_kernel<true> : fa::fa_fwd_fp8_kernel<false>;
  constexpr int smem = fa::Fp8Cfg::SMEM_BYTES;
  if ((st = ensure_smem(kern, dev, smem, causal ? done_c : done_nc, fa::kLaunchRegs)) != FA_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  mark_launch(s);
  fa::fa_fp8_transpose_v_kernel<<<dim3(static_cast<unsigned>((npad + 127) / 128), static_cast<unsigned>(H),
                                       static_cast<unsigned>(B)),
                                  128, 0, s>>>(static_cast<const uint8_t*>(v), static_cast<uint8_t*>(workspace), N,
                                               H, static_cast<int>(npad));
  if ((st = launch_status(s)) != FA_OK) return st;
  fa::Fp8Params p;
  p.o = o;
  p.lse = lse;
  p.B = B;
  p.N = N;
  p.H = H;
  p.npairs = (N + 255) / 256;
  p.group = head_group(static_cast<int64_t>(N) * 128 * 2, static_cast<int64_t>(B) * H);  // K and V^T bytes
  p.scale_log2 = scale * descale_q * descale_k * kLog2e;
  p.descale_v = descale_v;
  const int64_t grid = static_cast<int64_t>(p.npairs) * B * H;
  if (grid > 0x7fffffff) return FA_ERR_INVALID_ARG;
  kern<<<static_cast<unsigned>(grid), fa::Fp8Cfg::THREADS, smem, s>>>(mq, mk, mvt, p);
  return launch_status(s);
}

fa_status fa_record_launch_events(void* const* events, int n) {
  if (!events || n < 1 || n > 8) return FA_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i)
    if (!events[i]) return FA_ERR_INVALID_ARG;
  LaunchEvents& h = t_launch_events;
  for (int i = 0; i < n; ++i) h.ev[i] = static_cast<cudaEvent_t>(events[i]);
  h.n = n;
  h.used = 0;
  return FA_OK;
}

const char* fa_status_string(fa_status s) {
  switch (s) {
    case FA_OK: return "ok";
    case FA_ERR_INVALID_ARG: return "invalid argument (null/misaligned pointer or bad size)";
    case FA_ERR_UNSUPPORTED: return "unsupported (head dim must be 64 or 128; device must be sm_100)";
    case FA_ERR_CUDA: return "CUDA error";
    case FA_ERR_TIMEOUT: return "device pipeline wait timed out";
    case FA_ERR_WORKSPACE: return "workspace too small";
  }
  return "unknown status";
}

fa_status fa_get_device_error(void* stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_CUDA;
  }
  unsigned int word = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&word, fa::g_fa_error_word, sizeof(word)) != cudaSuccess ||
      cudaMemcpyToSymbol(fa::g_fa_error_word, &zero, sizeof(zero)) != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_CUDA;
  }
  if (word & fa::FA_DEVERR_TIMEOUT) return FA_ERR_TIMEOUT;
  return word ? FA_ERR_INVALID_ARG : FA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Backward pass without a caller-provided workspace.
//
// Some callers cannot allocate device memory at the point where they run the
// backward pass: code that executes inside a custom allocator or memory-pool
// callback, runtimes that forbid cudaMalloc after start-up (fixed memory
// budgets, pre-planned arenas), or plug-in hosts that hand out only the
// tensors themselves.  For them the scratch the backward pass needs (fp32 dQ
// accumulator and the D vector) lives in one statically sized device array
// that is part of this library's device image: every GPU that loads the
// library holds it until the process exits, and nothing is allocated per call.
//
// In host code `g_fa_static_scratch` names a host-side stand-in, not device
// memory, so the device address is looked up with cudaGetSymbolAddress once
// per device (on that device's first call, with the device current) and that
// address is what the kernels receive.  That first call per device performs
// the lookup and should therefore come before any stream capture.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kStaticScratchBytes = size_t(64) << 20;  // 64 MiB; matches FA_STATIC_SCRATCH_BYTES
static_assert(kStaticScratchBytes == FA_STATIC_SCRATCH_BYTES, "header and library disagree on the scratch size");

static __device__ __align__(256) unsigned char g_fa_static_scratch[kStaticScratchBytes];

void* g_static_scratch_ptr[kMaxDevices] = {};

fa_status static_scratch(int dev, void** out) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_static_scratch_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_fa_static_scratch) != cudaSuccess || ptr == nullptr) {
      cudaGetLastError();
      return FA_ERR_CUDA;
    }
    g_static_scratch_ptr[dev] = ptr;
  }
  *out = g_static_scratch_ptr[dev];
  return FA_OK;
}

}  // namespace

extern "C" fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                                    const void* dO, void* dq, void* dk, void* dv, int B, int N, int H, int d,
                                    float scale, int causal, void* stream) {
  LaunchEventsScope hook_scope;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (B < 1 || N < 1 || H < 1) return FA_ERR_INVALID_ARG;
  const size_t need = fa_bwd_workspace_size(B, N, H, d);
  if (need == 0) return FA_ERR_INVALID_ARG;
  if (need > kStaticScratchBytes) return FA_ERR_WORKSPACE;  // problem too large for the static scratch
  int dev;
  fa_status st = current_device(&dev);
  if (st != FA_OK) return st;
  void* scratch = nullptr;
  if ((st = static_scratch(dev, &scratch)) != FA_OK) return st;
  return fa_bwd(q, k, v, o, lse, dO, dq, dk, dv, scratch, kStaticScratchBytes, B, N, H, d, scale, causal, stream);
}

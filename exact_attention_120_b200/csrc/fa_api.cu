// Host side of the C ABI declared in include/fa.h: argument validation,
// TMA descriptor encoding, per-device set-up, the kernel launches, and the
// chunked copy pipeline of the host-buffer forward (fa_fwd_host).
//
// Nothing here computes any part of attention: every step runs in the
// kernels (fa_fwd_kernel and its instantiations, fa_combine_kernel for split
// keys, fa_bwd_kernel for the gradients).  There is no CPU fallback: without
// an sm_100 device the entry points return FA_ERR_UNSUPPORTED.

#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <initializer_list>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <utility>

#include "fa.h"
#include "fa_testing.h"
#include "fa_bwd_kernel.cuh"
#include "fa_combine.cuh"
#include "fa_fwd_kernel.cuh"

namespace {

// Device-side status word (FA_OK or FA_ERR_DEVICE_TIMEOUT), one per device.
__device__ int g_fa_status = 0;

// Workspace of fa_fwd_splitkv_noalloc: a fixed array in the module's device
// memory, so that entry point never allocates.  Every device that loads the
// library holds it until the process exits; all calls on a device share it.
// In host code the name only stands in for the symbol: its device address is
// taken with cudaGetSymbolAddress in the once-per-device set-up below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[FA_NOALLOC_SCRATCH_BYTES];

thread_local int t_last_cuda_error = 0;

constexpr unsigned long long kWaitTimeoutNs = 1000ull * 1000ull * 1000ull;  // 1 s per wait
constexpr int kMaxDevices = 64;
// fa_fwd_host: chunks of heads.  Measured on B=1, H=16, N=16384, d=128 from
// pinned memory: 4, 8, 16 chunks -> 4.73, 4.58, 4.54 ms per call.
constexpr int kHostChunks = 16;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

struct DeviceState {
  std::once_flag once;
  int status = FA_ERR_CUDA;  // result of the set-up
  int num_sms = 0;
  int* status_word = nullptr;     // device address of g_fa_status
  void* noalloc_scratch = nullptr;  // device address of g_noalloc_scratch
  // fa_fwd_host: one copy stream per direction and the events that order the
  // chunks, created on its first call on the device.  The mutex keeps the
  // enqueue of one call whole when several host threads call at once.
  std::once_flag host_once;
  int host_status = FA_ERR_CUDA;
  std::mutex host_mu;
  cudaStream_t copy_in = nullptr, copy_out = nullptr;
  cudaEvent_t ev_start = nullptr, ev_in_done = nullptr, ev_done = nullptr;
  cudaEvent_t ev_in[kHostChunks] = {}, ev_comp[kHostChunks] = {};
};

DeviceState g_dev[kMaxDevices];
std::once_flag g_encode_once;
EncodeTiledFn g_encode = nullptr;

int cuda_fail(cudaError_t e) {
  t_last_cuda_error = static_cast<int>(e);
  return FA_ERR_CUDA;
}

int setup_device(int dev, DeviceState& st) {
  cudaDeviceProp prop;
  cudaError_t e = cudaGetDeviceProperties(&prop, dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (prop.major != 10 || prop.minor != 0) return FA_ERR_UNSUPPORTED;  // sm_100 only
  st.num_sms = prop.multiProcessorCount;
  e = cudaFuncSetAttribute(fa::fa_fwd_kernel<fa::Cfg<64>>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           fa::Cfg<64>::kSmemBytes);
  if (e != cudaSuccess) return cuda_fail(e);
  e = cudaFuncSetAttribute(fa::fa_fwd_kernel<fa::Cfg<128>>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           fa::Cfg<128>::kSmemBytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(fa::fa_fwd_kernel<fa::Cfg<128, true>>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             fa::Cfg<128, true>::kSmemBytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(fa::fa_fwd_kernel<fa::Cfg<64>, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             fa::fwd_smem_bytes<fa::Cfg<64>, true>());
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(fa::fa_fwd_kernel<fa::Cfg<128>, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             fa::fwd_smem_bytes<fa::Cfg<128>, true>());
  if (e != cudaSuccess) return cuda_fail(e);
  e = cudaFuncSetAttribute(fa::fa_bwd_kernel<64, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           fa::BwdCfg<64>::kSmemBytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(fa::fa_bwd_kernel<128, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             fa::BwdCfg<128>::kSmemBytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(fa::fa_bwd_kernel<64, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             fa::BwdCfg<64>::kSmemBytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(fa::fa_bwd_kernel<128, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             fa::BwdCfg<128>::kSmemBytes);
  if (e != cudaSuccess) return cuda_fail(e);
  void* sym = nullptr;
  e = cudaGetSymbolAddress(&sym, g_fa_status);
  if (e != cudaSuccess) return cuda_fail(e);
  st.status_word = static_cast<int*>(sym);
  // With this device current: the device address of the no-allocation
  // workspace (loading the module above already reserved the array).
  sym = nullptr;
  e = cudaGetSymbolAddress(&sym, g_noalloc_scratch);
  if (e != cudaSuccess) return cuda_fail(e);
  st.noalloc_scratch = sym;
  return FA_OK;
}

int get_device_state(DeviceState** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
  DeviceState& st = g_dev[dev];
  std::call_once(st.once, [&] { st.status = setup_device(dev, st); });
  if (st.status != FA_OK) return st.status;
  *out = &st;
  return FA_OK;
}

int setup_host_streams(DeviceState& st) {
  cudaError_t e = cudaStreamCreateWithFlags(&st.copy_in, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&st.copy_out, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&st.ev_start, cudaEventDisableTiming);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&st.ev_in_done, cudaEventDisableTiming);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&st.ev_done, cudaEventDisableTiming);
  for (int c = 0; c < kHostChunks && e == cudaSuccess; ++c) {
    e = cudaEventCreateWithFlags(&st.ev_in[c], cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&st.ev_comp[c], cudaEventDisableTiming);
  }
  return e == cudaSuccess ? FA_OK : cuda_fail(e);
}

int get_encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  });
  return g_encode ? FA_OK : FA_ERR_CUDA;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Launch with programmatic stream serialization: the kernel may begin while
// the previous kernel on the stream finishes; every kernel of this library
// waits for that kernel (griddepcontrol.wait) before it touches global
// memory, so only its prologue overlaps (launch latency, tensor-memory
// allocation, barrier set-up).
// `overlap` = false launches the plain way (the kernel then starts after the
// previous one has finished).  Measured on one B200: overlap gains 7-12 % on
// forward launches of at most two rounds of work units (tiny 9.1 -> 8.1 us,
// small 21.2 -> 19.8 us) and on the backward (small 68.4 -> 63.4 us), and is
// neutral on long ones except variable-length batches, where it cost 7 %
// (CTAs placed in a different order on the SMs); so the forward uses it only
// for short grids.
template <class... Params, class... Args>
cudaError_t launch(bool overlap, void (*kernel)(Params...), unsigned grid, unsigned block, size_t smem,
                   cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = overlap ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// True if the pointer is device (or managed) memory the GPU can address.
bool is_device_pointer(const void* p) {
  cudaPointerAttributes attr;
  if (cudaPointerGetAttributes(&attr, p) != cudaSuccess) {
    cudaGetLastError();  // clear the sticky-free error state of the query
    return false;
  }
  return attr.type == cudaMemoryTypeDevice || attr.type == cudaMemoryTypeManaged;
}

// [B*H][N][d] bf16 (elt_bytes 2) or 8-bit (elt_bytes 1), boxes of 128 bytes
// x 128 rows, 128-byte swizzle.
int encode_qkv_map(CUtensorMap* map, const void* ptr, int BH, int N, int d, int elt_bytes = 2) {
  const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)BH};
  const cuuint64_t strides[2] = {(cuuint64_t)d * elt_bytes, (cuuint64_t)N * d * elt_bytes};
  const cuuint32_t box[3] = {(cuuint32_t)(128 / elt_bytes), 128, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUtensorMapDataType dt =
      elt_bytes == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  CUresult r = g_encode(map, dt, 3, const_cast<void*>(ptr), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    t_last_cuda_error = static_cast<int>(r);
    return FA_ERR_CUDA;
  }
  return FA_OK;
}

// Packed tokens [T][H][d] bf16 as a {d, H, T} map: a box of 64 columns x 1
// head x 128 tokens lands in shared memory as the same 128-row tile.
int encode_varlen_map(CUtensorMap* map, const void* ptr, int T, int H, int d) {
  const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)T};
  const cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2};
  const cuuint32_t box[3] = {64, 1, 128};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    t_last_cuda_error = static_cast<int>(r);
    return FA_ERR_CUDA;
  }
  return FA_OK;
}

constexpr int kMaxSplits = 256;

// Heads per group of the causal work order: as many as keep their K and V
// (2 x nk x d x elt_bytes each) within `budget_mb` of the 126 MB L2.  Dense
// batches use 96 MB: their heads all have the longest rows, and splitting
// them into more groups leaves a tail (mid-size causal: 1043 -> 855 TFLOP/s
// at 48 MB).  Variable-length batches use 48 MB: there the K/V of the long
// sequences were read from DRAM about four times over at 96 MB, and 48 MB
// measured 815 -> 889 TFLOP/s on a mix of 32 sequences.
int causal_group(long long bh, long long nk, int d, int elt_bytes, long long budget_mb = 96) {
  const long long kv = 2ll * std::max(nk, 1ll) * d * elt_bytes;
  const long long g = (budget_mb << 20) / kv;
  return (int)std::max(1ll, std::min(bh, g));
}

// Bytes of the split-key workspace: fp32 partial O [splits][rows][d] followed
// by fp32 partial lse [splits][rows].
size_t splitkv_workspace_bytes(size_t rows, int d, int splits) {
  return (size_t)splits * rows * ((size_t)d + 1) * sizeof(float);
}

// True if the byte ranges [a, a + na) and [b, b + nb) share a byte.
bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return na > 0 && nb > 0 && x < y + nb && y < x + na;
}

// A buffer and its size in bytes, for the overlap checks.
struct Span {
  const void* p;
  size_t bytes;
};

// True if any output overlaps any input or another output.  Inputs may
// overlap each other (they are only read).
bool outputs_alias(std::initializer_list<Span> outs, std::initializer_list<Span> ins) {
  for (const Span* o = outs.begin(); o != outs.end(); ++o) {
    for (const Span& i : ins)
      if (overlaps(o->p, o->bytes, i.p, i.bytes)) return true;
    for (const Span* o2 = o + 1; o2 != outs.end(); ++o2)
      if (overlaps(o->p, o->bytes, o2->p, o2->bytes)) return true;
  }
  return false;
}

// Work decomposition of a forward call, derived from its sizes.
struct FwdGeom {
  long long bh = 0, nqt = 0, nkt = 0, npairs = 0;
  int kt_per_split = 0, splits = 1;
  size_t rows = 0;       // B * H * Nq
  size_t workspace = 0;  // split-key workspace bytes (0 for one slice)
};

// Every check of a forward call that needs no CUDA call: pointers, sizes,
// scale, causal flag, head dim, alignment, aliasing and the slice count.
// Fills `g` on success.
int check_fwd_args(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                   int Nq, int Nk, int d, float scale, int causal, const uint8_t* block_mask,
                   int num_splits, bool fp8, float q_descale, float k_descale, float v_descale,
                   FwdGeom& g) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARGUMENT;
  if (fp8 && !(std::isfinite(q_descale) && q_descale > 0.f && std::isfinite(k_descale) &&
               k_descale > 0.f && std::isfinite(v_descale) && v_descale > 0.f))
    return FA_ERR_INVALID_ARGUMENT;
  if (fp8 && d != 128) return FA_ERR_UNSUPPORTED;
  if (B < 1 || H < 1 || Nq < 1 || Nk < 1) return FA_ERR_INVALID_ARGUMENT;
  if (!(std::isfinite(scale) && scale > 0.f)) return FA_ERR_INVALID_ARGUMENT;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARGUMENT;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4))
    return FA_ERR_INVALID_ARGUMENT;
  g.bh = (long long)B * H;
  g.nqt = (Nq + fa::kBM - 1) / fa::kBM;
  g.nkt = (Nk + fa::kBN - 1) / fa::kBN;
  g.npairs = (g.nqt + 1) / 2;
  if (g.bh > INT32_MAX || g.bh * g.npairs > INT32_MAX || (long long)Nq * d * 2 >= (1ll << 40) ||
      (long long)Nk * d * 2 >= (1ll << 40))
    return FA_ERR_UNSUPPORTED;  // 32-bit work indices and TMA stride limits
  g.rows = (size_t)g.bh * Nq;
  const size_t eb = fp8 ? 1 : 2;
  const size_t kv_bytes = (size_t)g.bh * Nk * d * eb;
  const Span ins[] = {{q, g.rows * d * eb}, {k, kv_bytes}, {v, kv_bytes},
                      {block_mask, block_mask ? (size_t)(g.bh * g.nqt * g.nkt) : 0}};
  if (outputs_alias({{o, g.rows * d * 2}, {lse, g.rows * sizeof(float)}},
                    {ins[0], ins[1], ins[2], ins[3]}))
    return FA_ERR_INVALID_ARGUMENT;
  if (num_splits < 1 || num_splits > kMaxSplits) return FA_ERR_INVALID_ARGUMENT;
  // Slices of kt_per_split key tiles; the last one is never empty.
  g.kt_per_split = (int)((g.nkt + num_splits - 1) / num_splits);
  g.splits = (int)((g.nkt + g.kt_per_split - 1) / g.kt_per_split);
  if (g.bh * g.npairs * g.splits > INT32_MAX) return FA_ERR_UNSUPPORTED;
  g.workspace = g.splits > 1 ? splitkv_workspace_bytes(g.rows, d, g.splits) : 0;
  return FA_OK;
}

// Descriptors and launch shared by the forward entry points.  `g` comes from
// check_fwd_args.  With more than one slice, `workspace` holds at least
// g.workspace bytes and overlaps none of the call's buffers.
int launch_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
               int Nq, int Nk, int d, float scale, int causal, const uint8_t* block_mask,
               void* cuda_stream, unsigned long long timeout_ns, int starve_producer,
               const FwdGeom& g, DeviceState* st, void* workspace = nullptr, bool fp8 = false,
               float q_descale = 1.f, float k_descale = 1.f, float v_descale = 1.f,
               bool allow_overlap = true) {
  const long long bh = g.bh, nqt = g.nqt, nkt = g.nkt, npairs = g.npairs;
  const int splits = g.splits, kt_per_split = g.kt_per_split;
  const size_t rows = g.rows;
  int rc = FA_OK;
  if (!is_device_pointer(q) || !is_device_pointer(k) || !is_device_pointer(v) ||
      !is_device_pointer(o) || !is_device_pointer(lse) ||
      (block_mask && !is_device_pointer(block_mask)) ||
      (splits > 1 && !is_device_pointer(workspace)))
    return FA_ERR_INVALID_ARGUMENT;
  if ((rc = get_encoder()) != FA_OK) return rc;

  // ---- parameters
  fa::KernelParams p;
  std::memset(&p, 0, sizeof(p));
  const int eb = fp8 ? 1 : 2;
  if ((rc = encode_qkv_map(&p.tm_q, q, (int)bh, Nq, d, eb)) != FA_OK) return rc;
  if ((rc = encode_qkv_map(&p.tm_k, k, (int)bh, Nk, d, eb)) != FA_OK) return rc;
  if ((rc = encode_qkv_map(&p.tm_v, v, (int)bh, Nk, d, eb)) != FA_OK) return rc;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.o_v8 = aligned(o, 32) ? 1 : 0;
  p.lse = lse;
  p.mask = block_mask;
  p.Nq = Nq;
  p.Nk = Nk;
  p.nqt = (int)nqt;
  p.nkt = (int)nkt;
  p.causal_off = Nk - Nq;
  p.npairs = (int)npairs;
  p.bh = (int)bh;
  p.group = causal_group(bh, Nk, d, eb);
  p.items = (int)(bh * npairs * splits);
  p.splits = splits;
  p.kt_per_split = kt_per_split;
  if (splits > 1) {
    p.part_o = static_cast<float*>(workspace);
    p.part_lse = p.part_o + (size_t)splits * rows * d;
  }
  p.causal = causal;
  p.scale_log2 = (float)((double)scale * q_descale * k_descale * 1.4426950408889634074);
  p.o_scale = v_descale;
  p.timeout_ns = timeout_ns;
  p.status = st->status_word;
  p.starve_producer = starve_producer;

  // ---- launch: persistent grid, one CTA per SM
  const int grid = p.items < st->num_sms ? p.items : st->num_sms;
  cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
  const bool overlap = allow_overlap && p.items <= 2 * st->num_sms;  // short grids: launch overlap pays
  cudaError_t e;
  if (fp8)
    e = launch(overlap, fa::fa_fwd_kernel<fa::Cfg<128, true>>, grid, fa::kThreads, fa::Cfg<128, true>::kSmemBytes, stream, p);
  else if (d == 64)
    e = launch(overlap, fa::fa_fwd_kernel<fa::Cfg<64>>, grid, fa::kThreads, fa::Cfg<64>::kSmemBytes, stream, p);
  else
    e = launch(overlap, fa::fa_fwd_kernel<fa::Cfg<128>>, grid, fa::kThreads, fa::Cfg<128>::kSmemBytes, stream, p);
  if (e != cudaSuccess) return cuda_fail(e);
  if (splits > 1) {  // merge the slices (concatenated-softmax rule)
    const unsigned blocks = (unsigned)((rows * 32 + 255) / 256);
    const float* po = p.part_o;
    const float* pl = p.part_lse;
    __nv_bfloat16* ob = static_cast<__nv_bfloat16*>(o);
    const long long nrows = (long long)rows;
    if (d == 64)
      e = launch(true, fa::fa_combine_kernel<64>, blocks, 256, 0, stream, po, pl, ob, lse, nrows, splits);
    else
      e = launch(true, fa::fa_combine_kernel<128>, blocks, 256, 0, stream, po, pl, ob, lse, nrows, splits);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  return FA_OK;
}

// A forward call with a caller workspace (or none): host checks, then the
// device set-up, then the launch.
int run_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Nq,
            int Nk, int d, float scale, int causal, const uint8_t* block_mask, void* cuda_stream,
            unsigned long long timeout_ns, int starve_producer, int num_splits = 1,
            void* workspace = nullptr, size_t workspace_bytes = 0, bool fp8 = false,
            float q_descale = 1.f, float k_descale = 1.f, float v_descale = 1.f) {
  FwdGeom g;
  int rc = check_fwd_args(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal, block_mask, num_splits,
                          fp8, q_descale, k_descale, v_descale, g);
  if (rc != FA_OK) return rc;
  if (g.splits > 1) {
    const size_t eb = fp8 ? 1 : 2;
    const size_t kv_bytes = (size_t)g.bh * Nk * d * eb;
    if (!workspace || !aligned(workspace, 16) || workspace_bytes < g.workspace ||
        outputs_alias({{workspace, g.workspace}},
                      {{q, g.rows * d * eb}, {k, kv_bytes}, {v, kv_bytes}, {o, g.rows * d * 2},
                       {lse, g.rows * sizeof(float)},
                       {block_mask, block_mask ? (size_t)(g.bh * g.nqt * g.nkt) : 0}}))
      return FA_ERR_INVALID_ARGUMENT;
  }
  DeviceState* st = nullptr;
  if ((rc = get_device_state(&st)) != FA_OK) return rc;
  return launch_fwd(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal, block_mask, cuda_stream,
                    timeout_ns, starve_producer, g, st, workspace, fp8, q_descale, k_descale,
                    v_descale);
}

}  // namespace

extern "C" {

int fa_fwd_stream(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                  int N, int d, float scale, int causal, const uint8_t* block_mask,
                  void* cuda_stream) {
  return run_fwd(q, k, v, o, lse, B, H, N, N, d, scale, causal, block_mask, cuda_stream,
                 kWaitTimeoutNs, 0);
}

int fa_fwd_qk(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
              int Nq, int Nk, int d, float scale, int causal, const uint8_t* block_mask,
              void* cuda_stream) {
  return run_fwd(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal, block_mask, cuda_stream,
                 kWaitTimeoutNs, 0);
}

size_t fa_fwd_splitkv_workspace_bytes(int B, int H, int Nq, int Nk, int d, int num_splits) {
  if (B < 1 || H < 1 || Nq < 1 || Nk < 1 || num_splits < 1 || num_splits > kMaxSplits) return 0;
  const long long nkt = (Nk + fa::kBN - 1) / fa::kBN;
  const long long per = (nkt + num_splits - 1) / num_splits;
  const int splits = (int)((nkt + per - 1) / per);
  return splits > 1 ? splitkv_workspace_bytes((size_t)B * H * Nq, d, splits) : 0;
}

int fa_fwd_splitkv_heuristic(int B, int H, int Nq, int Nk) {
  DeviceState* st = nullptr;
  if (B < 1 || H < 1 || Nq < 1 || Nk < 1 || get_device_state(&st) != FA_OK) return 1;
  const long long units = (long long)B * H * (((Nq + fa::kBM - 1) / fa::kBM + 1) / 2);
  const long long nkt = (Nk + fa::kBN - 1) / fa::kBN;
  if (units >= st->num_sms || nkt < 4) return 1;
  // About two waves of units, each slice at least two key tiles long.
  long long splits = (2 * st->num_sms + units - 1) / units;
  if (splits > nkt / 2) splits = nkt / 2;
  if (splits > kMaxSplits) splits = kMaxSplits;
  return splits < 1 ? 1 : (int)splits;
}

int fa_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                   int Nq, int Nk, int d, float scale, int causal, const uint8_t* block_mask,
                   int num_splits, void* workspace, size_t workspace_bytes, void* cuda_stream) {
  return run_fwd(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal, block_mask, cuda_stream,
                 kWaitTimeoutNs, 0, num_splits, workspace, workspace_bytes);
}

int fa_fwd_splitkv_noalloc(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                           int H, int Nq, int Nk, int d, float scale, int causal,
                           const uint8_t* block_mask, int num_splits, void* cuda_stream) {
  // Every host-side check first, with no CUDA call; then the size limit.
  FwdGeom g;
  int rc = check_fwd_args(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal, block_mask, num_splits,
                          false, 1.f, 1.f, 1.f, g);
  if (rc != FA_OK) return rc;
  if (g.workspace > (size_t)FA_NOALLOC_SCRATCH_BYTES) return FA_ERR_UNSUPPORTED;
  // The once-per-device set-up (the first library call on this device) took
  // the array's device address with this device current.
  DeviceState* st = nullptr;
  if ((rc = get_device_state(&st)) != FA_OK) return rc;
  // The split kernel writes every partial it later reads (empty slices
  // included), so nothing in the array has to start at zero.  The array is
  // the library's own memory: it cannot overlap the caller's buffers.
  return launch_fwd(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal, block_mask, cuda_stream,
                    kWaitTimeoutNs, 0, g, st, g.splits > 1 ? st->noalloc_scratch : nullptr);
}

size_t fa_bwd_workspace_bytes(int B, int H, int Nq) {
  if (B < 1 || H < 1 || Nq < 1) return 0;
  return ((size_t)B * H * Nq * sizeof(float) + 15) / 16 * 16;
}

int fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
           const void* dout, void* dq, void* dk, void* dv, int B, int H, int Nq, int Nk, int d,
           float scale, int causal, const uint8_t* block_mask, void* workspace,
           size_t workspace_bytes, void* cuda_stream) {
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv || !workspace)
    return FA_ERR_INVALID_ARGUMENT;
  if (B < 1 || H < 1 || Nq < 1 || Nk < 1) return FA_ERR_INVALID_ARGUMENT;
  if (!(std::isfinite(scale) && scale > 0.f)) return FA_ERR_INVALID_ARGUMENT;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARGUMENT;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  for (const void* ptr : std::initializer_list<const void*>{q, k, v, o, dout, dq, dk, dv, workspace})
    if (!aligned(ptr, 16)) return FA_ERR_INVALID_ARGUMENT;
  if (!aligned(lse, 4)) return FA_ERR_INVALID_ARGUMENT;
  const long long bh = (long long)B * H;
  const long long nqt = (Nq + fa::kBM - 1) / fa::kBM;
  const long long nkt = (Nk + fa::kBN - 1) / fa::kBN;
  if (bh * nqt > INT32_MAX || bh * nkt > INT32_MAX || (long long)Nq * d * 2 >= (1ll << 40) ||
      (long long)Nk * d * 2 >= (1ll << 40))
    return FA_ERR_UNSUPPORTED;
  const size_t ws_need = fa_bwd_workspace_bytes(B, H, Nq);
  if (workspace_bytes < ws_need) return FA_ERR_INVALID_ARGUMENT;
  {
    const size_t qb = (size_t)bh * Nq * d * 2, kb = (size_t)bh * Nk * d * 2;
    if (outputs_alias({{dq, qb}, {dk, kb}, {dv, kb}, {workspace, ws_need}},
                      {{q, qb}, {k, kb}, {v, kb}, {o, qb}, {lse, (size_t)bh * Nq * sizeof(float)},
                       {dout, qb}, {block_mask, block_mask ? (size_t)(bh * nqt * nkt) : 0}}))
      return FA_ERR_INVALID_ARGUMENT;
  }

  DeviceState* st = nullptr;
  int rc = get_device_state(&st);
  if (rc != FA_OK) return rc;
  for (const void* ptr :
       std::initializer_list<const void*>{q, k, v, o, lse, dout, dq, dk, dv, workspace})
    if (!is_device_pointer(ptr)) return FA_ERR_INVALID_ARGUMENT;
  if (block_mask && !is_device_pointer(block_mask)) return FA_ERR_INVALID_ARGUMENT;
  if ((rc = get_encoder()) != FA_OK) return rc;

  fa::BwdParams p;
  std::memset(&p, 0, sizeof(p));
  if ((rc = encode_qkv_map(&p.tm_q, q, (int)bh, Nq, d)) != FA_OK) return rc;
  if ((rc = encode_qkv_map(&p.tm_k, k, (int)bh, Nk, d)) != FA_OK) return rc;
  if ((rc = encode_qkv_map(&p.tm_v, v, (int)bh, Nk, d)) != FA_OK) return rc;
  if ((rc = encode_qkv_map(&p.tm_do, dout, (int)bh, Nq, d)) != FA_OK) return rc;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.o = static_cast<const __nv_bfloat16*>(o);
  p.dout = static_cast<const __nv_bfloat16*>(dout);
  p.lse = lse;
  p.delta = static_cast<float*>(workspace);
  p.dq = static_cast<__nv_bfloat16*>(dq);
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dv = static_cast<__nv_bfloat16*>(dv);
  p.mask = block_mask;
  p.Nq = Nq;
  p.Nk = Nk;
  p.nqt = (int)nqt;
  p.nkt = (int)nkt;
  p.causal_off = Nk - Nq;
  p.bh = (int)bh;
  p.causal = causal;
  p.scale = scale;
  p.scale_log2 = (float)((double)scale * 1.4426950408889634074);
  p.timeout_ns = kWaitTimeoutNs;
  p.status = st->status_word;

  cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
  const int grid_q = (int)std::min<long long>(bh * nqt, st->num_sms);
  const int grid_k = (int)std::min<long long>(bh * nkt, st->num_sms);
  cudaError_t e;
  if (d == 64) {
    e = launch(true, fa::fa_bwd_kernel<64, true>, grid_q, fa::kBwdThreads, fa::BwdCfg<64>::kSmemBytes, stream, p);
    if (e == cudaSuccess)
      e = launch(true, fa::fa_bwd_kernel<64, false>, grid_k, fa::kBwdThreads, fa::BwdCfg<64>::kSmemBytes, stream, p);
  } else {
    e = launch(true, fa::fa_bwd_kernel<128, true>, grid_q, fa::kBwdThreads, fa::BwdCfg<128>::kSmemBytes, stream, p);
    if (e == cudaSuccess)
      e = launch(true, fa::fa_bwd_kernel<128, false>, grid_k, fa::kBwdThreads, fa::BwdCfg<128>::kSmemBytes, stream, p);
  }
  if (e != cudaSuccess) return cuda_fail(e);
  return FA_OK;
}

int fa_testing_fwd_starved(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                           int H, int N, int d, float scale, int causal,
                           const uint8_t* block_mask, void* cuda_stream,
                           unsigned long long timeout_ns) {
  if (timeout_ns == 0 || timeout_ns > kWaitTimeoutNs) return FA_ERR_INVALID_ARGUMENT;
  return run_fwd(q, k, v, o, lse, B, H, N, N, d, scale, causal, block_mask, cuda_stream,
                 timeout_ns, 1);
}

int fa_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
               int Nq, int Nk, int d, float scale, int causal, const uint8_t* block_mask,
               float q_descale, float k_descale, float v_descale, void* cuda_stream) {
  return run_fwd(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal, block_mask, cuda_stream,
                 kWaitTimeoutNs, 0, 1, nullptr, 0, true, q_descale, k_descale, v_descale);
}

int fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                  const int* cu_seqlens_q, const int* cu_seqlens_k, int B, int H, int total_q,
                  int total_k, int max_seqlen_q, int d, float scale, int causal,
                  void* cuda_stream) {
  if (!q || !k || !v || !o || !lse || !cu_seqlens_q || !cu_seqlens_k) return FA_ERR_INVALID_ARGUMENT;
  if (B < 1 || H < 1 || total_q < 1 || total_k < 1 || max_seqlen_q < 1) return FA_ERR_INVALID_ARGUMENT;
  if (!(std::isfinite(scale) && scale > 0.f)) return FA_ERR_INVALID_ARGUMENT;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARGUMENT;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4) ||
      !aligned(cu_seqlens_q, 4) || !aligned(cu_seqlens_k, 4))
    return FA_ERR_INVALID_ARGUMENT;
  const long long bh = (long long)B * H;
  const long long nqt = (max_seqlen_q + fa::kBM - 1) / fa::kBM;
  const long long npairs = (nqt + 1) / 2;
  if (bh * npairs > INT32_MAX || (long long)total_q * H > INT32_MAX) return FA_ERR_UNSUPPORTED;
  {
    const size_t qb = (size_t)total_q * H * d * 2, kb = (size_t)total_k * H * d * 2;
    const size_t cb = ((size_t)B + 1) * sizeof(int);
    if (outputs_alias({{o, qb}, {lse, (size_t)total_q * H * sizeof(float)}},
                      {{q, qb}, {k, kb}, {v, kb}, {cu_seqlens_q, cb}, {cu_seqlens_k, cb}}))
      return FA_ERR_INVALID_ARGUMENT;
  }

  DeviceState* st = nullptr;
  int rc = get_device_state(&st);
  if (rc != FA_OK) return rc;
  for (const void* ptr : std::initializer_list<const void*>{q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k})
    if (!is_device_pointer(ptr)) return FA_ERR_INVALID_ARGUMENT;
  if ((rc = get_encoder()) != FA_OK) return rc;

  fa::KernelParams p;
  std::memset(&p, 0, sizeof(p));
  p.o = static_cast<__nv_bfloat16*>(o);
  p.o_v8 = aligned(o, 32) ? 1 : 0;
  p.lse = lse;
  p.mask = nullptr;
  p.Nq = max_seqlen_q;
  p.Nk = total_k;
  p.nqt = (int)nqt;
  p.nkt = (total_k + fa::kBN - 1) / fa::kBN;
  p.causal_off = 0;
  p.npairs = (int)npairs;
  p.splits = 1;
  p.kt_per_split = p.nkt;
  p.causal = causal;
  p.scale_log2 = (float)((double)scale * 1.4426950408889634074);
  p.o_scale = 1.0f;
  p.timeout_ns = kWaitTimeoutNs;
  p.status = st->status_word;
  p.heads = H;
  p.total_q = total_q;
  p.total_k = total_k;
  // Causal order: the heads of one sequence are taken in groups whose K/V
  // together fill at most 48 MiB of L2.
  p.group_keys = (int)((48ll << 20) / (2ll * d * 2));
  if ((rc = encode_varlen_map(&p.tm_q, q, total_q, H, d)) != FA_OK) return rc;
  if ((rc = encode_varlen_map(&p.tm_k, k, total_k, H, d)) != FA_OK) return rc;
  if ((rc = encode_varlen_map(&p.tm_v, v, total_k, H, d)) != FA_OK) return rc;
  // One launch per fa::kMaxVarlenSeqs sequences (the kernel's table of their
  // first work units); the offsets are absolute, so a later launch only
  // starts further into cu_seqlens.  The kernel deals the units that exist;
  // the grid is sized by the bound max_seqlen_q gives.
  cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
  for (int b0 = 0; b0 < B; b0 += fa::kMaxVarlenSeqs) {
    const int nseq = std::min(B - b0, fa::kMaxVarlenSeqs);
    p.cu_q = cu_seqlens_q + b0;
    p.cu_k = cu_seqlens_k + b0;
    p.nseq = nseq;
    p.bh = nseq * H;
    p.items = (int)(p.bh * npairs);
    const int grid = p.items < st->num_sms ? p.items : st->num_sms;
    const bool overlap = p.items <= 2 * st->num_sms;
    cudaError_t e;
    if (d == 64)
      e = launch(overlap, fa::fa_fwd_kernel<fa::Cfg<64>, true>, grid, fa::kThreads,
                 fa::fwd_smem_bytes<fa::Cfg<64>, true>(), stream, p);
    else
      e = launch(overlap, fa::fa_fwd_kernel<fa::Cfg<128>, true>, grid, fa::kThreads,
                 fa::fwd_smem_bytes<fa::Cfg<128>, true>(), stream, p);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  return FA_OK;
}

int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N,
           int d, float scale, int causal, const uint8_t* block_mask) {
  return fa_fwd_stream(q, k, v, o, lse, B, H, N, d, scale, causal, block_mask, nullptr);
}

int fa_fwd_host(const void* q_host, const void* k_host, const void* v_host, void* o_host,
                float* lse_host, void* q_dev, void* k_dev, void* v_dev, void* o_dev, float* lse_dev,
                int B, int H, int N, int d, float scale, int causal, const uint8_t* block_mask,
                void* cuda_stream) {
  // Host checks first, with no CUDA call.
  if (!q_host || !k_host || !v_host || !o_host || !lse_host) return FA_ERR_INVALID_ARGUMENT;
  FwdGeom g;
  int rc = check_fwd_args(q_dev, k_dev, v_dev, o_dev, lse_dev, B, H, N, N, d, scale, causal,
                          block_mask, 1, false, 1.f, 1.f, 1.f, g);
  if (rc != FA_OK) return rc;
  const size_t head_bytes = (size_t)N * d * 2;  // one head of Q, K, V or O
  const size_t qkv_bytes = (size_t)g.bh * head_bytes;
  if (outputs_alias({{o_host, qkv_bytes}, {lse_host, g.rows * sizeof(float)}},
                    {{q_host, qkv_bytes}, {k_host, qkv_bytes}, {v_host, qkv_bytes}}))
    return FA_ERR_INVALID_ARGUMENT;

  DeviceState* st = nullptr;
  if ((rc = get_device_state(&st)) != FA_OK) return rc;
  for (const void* ptr : std::initializer_list<const void*>{q_dev, k_dev, v_dev, o_dev, lse_dev})
    if (!is_device_pointer(ptr)) return FA_ERR_INVALID_ARGUMENT;
  if (block_mask && !is_device_pointer(block_mask)) return FA_ERR_INVALID_ARGUMENT;
  for (const void* ptr : std::initializer_list<const void*>{q_host, k_host, v_host, o_host, lse_host})
    if (is_device_pointer(ptr)) return FA_ERR_INVALID_ARGUMENT;
  std::call_once(st->host_once, [&] { st->host_status = setup_host_streams(*st); });
  if (st->host_status != FA_OK) return st->host_status;
  std::lock_guard<std::mutex> lock(st->host_mu);

  // Chunk c of whole heads [h0, h0 + hn): copy in on copy_in, compute on the
  // caller's stream once its copy has landed, copy out on copy_out once it is
  // computed.  Each chunk is a batch of hn heads for the kernel.
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  const long long nchunks = std::min<long long>(kHostChunks, g.bh);
  const long long per = (g.bh + nchunks - 1) / nchunks;
  const size_t mask_head = (size_t)g.nqt * g.nkt;
  cudaError_t e = cudaEventRecord(st->ev_start, s);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(st->copy_in, st->ev_start, 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(st->copy_out, st->ev_start, 0);
  if (e != cudaSuccess) return cuda_fail(e);
  int c = 0;
  for (long long h0 = 0; h0 < g.bh && e == cudaSuccess && rc == FA_OK; h0 += per, ++c) {
    const int hn = (int)std::min(per, g.bh - h0);
    const size_t off = (size_t)h0 * head_bytes, bytes = (size_t)hn * head_bytes;
    const size_t loff = (size_t)h0 * N * sizeof(float), lbytes = (size_t)hn * N * sizeof(float);
    char* qd = static_cast<char*>(q_dev) + off;
    char* kd = static_cast<char*>(k_dev) + off;
    char* vd = static_cast<char*>(v_dev) + off;
    char* od = static_cast<char*>(o_dev) + off;
    float* ld = reinterpret_cast<float*>(reinterpret_cast<char*>(lse_dev) + loff);
    e = cudaMemcpyAsync(qd, static_cast<const char*>(q_host) + off, bytes, cudaMemcpyHostToDevice, st->copy_in);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(kd, static_cast<const char*>(k_host) + off, bytes, cudaMemcpyHostToDevice, st->copy_in);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(vd, static_cast<const char*>(v_host) + off, bytes, cudaMemcpyHostToDevice, st->copy_in);
    if (e == cudaSuccess) e = cudaEventRecord(st->ev_in[c], st->copy_in);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s, st->ev_in[c], 0);
    if (e != cudaSuccess) break;
    FwdGeom gc;
    const uint8_t* mc = block_mask ? block_mask + (size_t)h0 * mask_head : nullptr;
    rc = check_fwd_args(qd, kd, vd, od, ld, 1, hn, N, N, d, scale, causal, mc, 1, false, 1.f, 1.f, 1.f, gc);
    if (rc == FA_OK)
      rc = launch_fwd(qd, kd, vd, od, ld, 1, hn, N, N, d, scale, causal, mc, s, kWaitTimeoutNs, 0, gc, st,
                      nullptr, false, 1.f, 1.f, 1.f, /*allow_overlap=*/false);
    if (rc != FA_OK) break;
    e = cudaEventRecord(st->ev_comp[c], s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(st->copy_out, st->ev_comp[c], 0);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(static_cast<char*>(o_host) + off, od, bytes, cudaMemcpyDeviceToHost, st->copy_out);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(reinterpret_cast<char*>(lse_host) + loff, ld, lbytes, cudaMemcpyDeviceToHost,
                          st->copy_out);
  }
  // Whatever was enqueued, the caller's stream waits for both copy streams,
  // so that no copy of this call outlives it unordered.
  cudaError_t e2 = cudaEventRecord(st->ev_done, st->copy_out);
  if (e2 == cudaSuccess) e2 = cudaStreamWaitEvent(s, st->ev_done, 0);
  if (e2 == cudaSuccess) e2 = cudaEventRecord(st->ev_in_done, st->copy_in);
  if (e2 == cudaSuccess) e2 = cudaStreamWaitEvent(s, st->ev_in_done, 0);
  if (e != cudaSuccess) return cuda_fail(e);
  if (rc != FA_OK) return rc;
  if (e2 != cudaSuccess) return cuda_fail(e2);
  return FA_OK;
}

int fa_device_status(void* cuda_stream) {
  DeviceState* st = nullptr;
  int rc = get_device_state(&st);
  if (rc != FA_OK) return rc;
  cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
  int value = 0;
  cudaError_t e = cudaMemcpyAsync(&value, st->status_word, sizeof(int), cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(st->status_word, 0, sizeof(int), stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_fail(e);
  return value == 0 ? FA_OK : value;
}

const char* fa_status_string(int status) {
  switch (status) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARGUMENT: return "FA_ERR_INVALID_ARGUMENT";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED";
    case FA_ERR_CUDA: return "FA_ERR_CUDA";
    case FA_ERR_DEVICE_TIMEOUT: return "FA_ERR_DEVICE_TIMEOUT";
    default: return "FA_UNKNOWN_STATUS";
  }
}

int fa_last_cuda_error(void) { return t_last_cuda_error; }

int fa_launches_per_call(void) { return 1; }

}  // extern "C"

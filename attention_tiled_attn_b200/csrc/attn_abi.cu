// The C ABI (include/attn_b200.h): argument validation, dispatch between the
// prefill, decode and fp32 paths, the decode workspace, and the device
// status word.  Everything here is host code; the kernels live in the
// *_sm100.cu / fp32_simt.cu files.

#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "attn_b200.h"
#include "kernels.h"

namespace attn {

void* tensor_map_encoder() {
  static void* fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = p;
  });
  return fn;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

bool make_map_rows(void* map, const void* base, int dim, long long rows, long long heads, int box_rows) {
  auto fn = reinterpret_cast<EncodeTiledFn>(tensor_map_encoder());
  if (!fn) return false;
  cuuint64_t gdim[3] = {static_cast<cuuint64_t>(dim), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(heads)};
  cuuint64_t gstride[2] = {static_cast<cuuint64_t>(dim) * 2, static_cast<cuuint64_t>(rows) * dim * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estride[3] = {1, 1, 1};
  const CUresult r = fn(static_cast<CUtensorMap*>(map), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base),
                        gdim, gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

namespace {

constexpr int MAX_DEVICES = 64;

struct Workspace {
  void* ptr = nullptr;
  size_t bytes = 0;
};

std::mutex g_mutex;
Workspace g_ws[MAX_DEVICES];
int g_fail_allocs = 0;  // failure-path check: workspace allocations still to refuse (under g_mutex)
int g_num_sms[MAX_DEVICES] = {0};
int g_cc_major[MAX_DEVICES] = {0};

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int device_info(int* dev, int* sms, int* major) {
  if (cudaGetDevice(dev) != cudaSuccess || *dev < 0 || *dev >= MAX_DEVICES) return ATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_num_sms[*dev] == 0) {
    int s = 0, m = 0;
    if (cudaDeviceGetAttribute(&s, cudaDevAttrMultiProcessorCount, *dev) != cudaSuccess) return ATTN_ERR_CUDA;
    if (cudaDeviceGetAttribute(&m, cudaDevAttrComputeCapabilityMajor, *dev) != cudaSuccess) return ATTN_ERR_CUDA;
    g_num_sms[*dev] = s;
    g_cc_major[*dev] = m;
  }
  *sms = g_num_sms[*dev];
  *major = g_cc_major[*dev];
  return ATTN_OK;
}

// Grows the library-owned decode workspace of `dev` to at least `bytes`, stream-ordered.
int ensure_workspace(int dev, size_t bytes, cudaStream_t stream, void** out) {
  std::lock_guard<std::mutex> lock(g_mutex);
  Workspace& w = g_ws[dev];
  if (w.bytes < bytes) {
    if (g_fail_allocs > 0) {  // an injected allocation failure: the same return as a failed cudaMallocAsync
      --g_fail_allocs;
      return ATTN_ERR_WORKSPACE;
    }
    if (w.ptr) cudaFreeAsync(w.ptr, stream);
    w.ptr = nullptr;
    w.bytes = 0;
    void* p = nullptr;
    if (cudaMallocAsync(&p, bytes, stream) != cudaSuccess) {
      cudaGetLastError();
      return ATTN_ERR_WORKSPACE;
    }
    w.ptr = p;
    w.bytes = bytes;
  }
  *out = w.ptr;
  return ATTN_OK;
}

}  // namespace

// Checks shared by every entry point (after each has checked its mask arguments).
int validate(const void* q, const void* k, const void* v, void* out, float* lse, int N, int Hq, int H, int L, int S,
             int E, int Ev, float scale, int mode, const float* sink_logits, const float* bias, int dtype) {
  if (!q || !k || !v || !out) return ATTN_ERR_NULL_POINTER;
  if (N < 1 || Hq < 1 || H < 1 || L < 1 || S < 1) return ATTN_ERR_BAD_SHAPE;
  if (Hq % H != 0) return ATTN_ERR_GQA;
  if ((E != 64 && E != 128) || (Ev != 64 && Ev != 128)) return ATTN_ERR_HEAD_DIM;
  if (!std::isfinite(scale) || scale <= 0.f) return ATTN_ERR_SCALE;
  if (mode < ATTN_DOT || mode > ATTN_SINK) return ATTN_ERR_MODE;
  if (mode == ATTN_SINK && sink_logits == nullptr) return ATTN_ERR_SINK;
  if (dtype != ATTN_BF16 && dtype != ATTN_FP32) return ATTN_ERR_DTYPE;
  // every element offset must fit the kernels' 64-bit indexing and the per-head
  // row index their 32-bit coordinates; the fp32 grid holds N*Hq in gridDim.y
  const long long NHq = static_cast<long long>(N) * Hq;
  const long long NH = static_cast<long long>(N) * H;
  if (NHq > (1LL << 31) - 1 || NH > (1LL << 31) - 1) return ATTN_ERR_BAD_SHAPE;
  if (NHq * L > (1LL << 40) || NH * S > (1LL << 40)) return ATTN_ERR_BAD_SHAPE;
  if (dtype == ATTN_FP32 && NHq > 65535) return ATTN_ERR_BAD_SHAPE;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16)) return ATTN_ERR_ALIGNMENT;
  if (bias && !aligned(bias, 16)) return ATTN_ERR_ALIGNMENT;
  if (lse && !aligned(lse, 4)) return ATTN_ERR_ALIGNMENT;
  if (sink_logits && !aligned(sink_logits, 4)) return ATTN_ERR_ALIGNMENT;
  return ATTN_OK;
}

AttnArgs make_args(const void* q, const void* k, const void* v, void* out, float* lse, int N, int Hq, int H, int L,
                   int S, int E, int Ev, float scale, int mode, const float* sink_logits, int mask_kind, int window,
                   int keep, const float* bias, const uint32_t* mask_bits = nullptr, const int* kv_start = nullptr,
                   const int* kv_end = nullptr) {
  AttnArgs a{};
  a.mask_bits = mask_bits;
  a.kv_start = kv_start;
  a.kv_end = kv_end;
  a.q = q;
  a.k = k;
  a.v = v;
  a.out = out;
  a.lse = lse;
  a.N = N;
  a.Hq = Hq;
  a.H = H;
  a.L = L;
  a.S = S;
  a.E = E;
  a.Ev = Ev;
  a.scale = scale;
  a.rbf = (mode == ATTN_RBF);
  a.sink = sink_logits;
  a.mask_kind = mask_kind;
  a.window = window;
  a.keep = keep;
  a.bias = bias;
  return a;
}

// Shared by the public entry points once they have checked their mask arguments:
// validates the rest and dispatches (fp32 kernel, split-key decode, tcgen05 prefill).
int forward(const void* q, const void* k, const void* v, void* out, float* lse, int N, int Hq, int H, int L, int S,
            int E, int Ev, float scale, int mode, const float* sink_logits, int mask_kind, int window, int keep,
            const float* bias, int dtype, void* stream_ptr, const uint32_t* mask_bits = nullptr,
            const int* kv_start = nullptr, const int* kv_end = nullptr) {
  const int st = validate(q, k, v, out, lse, N, Hq, H, L, S, E, Ev, scale, mode, sink_logits, bias, dtype);
  if (st != ATTN_OK) return st;
  int dev = 0, sms = 0, major = 0;
  if (device_info(&dev, &sms, &major) != ATTN_OK) return ATTN_ERR_CUDA;
  if (major != 10) return ATTN_ERR_DEVICE;
  const AttnArgs a = make_args(q, k, v, out, lse, N, Hq, H, L, S, E, Ev, scale, mode, sink_logits, mask_kind, window,
                               keep, bias, mask_bits, kv_start, kv_end);
  cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);

  if (dtype == ATTN_FP32) return launch_fp32(a, stream);
  if (decode_eligible(a)) {
    void* ws = nullptr;
    const size_t need = decode_workspace_bytes(a, sms);
    const int st = ensure_workspace(dev, need, stream, &ws);
    if (st != ATTN_OK) return st;
    return launch_decode_bf16(a, ws, need, sms, stream);
  }
  void* ws = nullptr;
  const size_t need = prefill_workspace_bytes(a);
  if (need > 0) {
    const int st2 = ensure_workspace(dev, need, stream, &ws);
    if (st2 != ATTN_OK) return st2;
  }
  return launch_prefill_bf16(a, ws, need, stream);
}

}  // namespace attn

extern "C" {

int attn_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int N, int Hq, int H, int L,
             int S, int E, int Ev, float scale, int mode, const float* sink_logits, int mask_kind, int window,
             const float* bias, int dtype, void* stream_ptr) {
  if (mask_kind < ATTN_MASK_NONE || mask_kind > ATTN_MASK_SLIDING_WINDOW) return ATTN_ERR_MASK;
  if (mask_kind == ATTN_MASK_SLIDING_WINDOW && window < 1) return ATTN_ERR_WINDOW;
  return attn::forward(q, k, v, out, lse, N, Hq, H, L, S, E, Ev, scale, mode, sink_logits, mask_kind, window, 0,
                       bias, dtype, stream_ptr);
}

int attn_fwd_streaming(const void* q, const void* k, const void* v, void* out, float* lse, int N, int Hq, int H,
                       int L, int S, int E, int Ev, float scale, int mode, const float* sink_logits, int window,
                       int keep_first, const float* bias, int dtype, void* stream_ptr) {
  if (window < 1) return ATTN_ERR_WINDOW;
  if (keep_first < 0) return ATTN_ERR_KEEP;
  return attn::forward(q, k, v, out, lse, N, Hq, H, L, S, E, Ev, scale, mode, sink_logits, attn::MASK_STREAM,
                       window, keep_first, bias, dtype, stream_ptr);
}

int attn_bwd(const void* q, const void* k, const void* v, const void* out, const void* dout, const float* lse,
             float* dq, float* dk, float* dv, float* dsink, int N, int Hq, int H, int L, int S, int E, int Ev,
             float scale, int mode, const float* sink_logits, int mask_kind, int window, int keep_first,
             const unsigned int* mask_bits, const int* kv_start, const int* kv_end, void* stream_ptr) {
  using namespace attn;
  if (!out || !dout || !lse || !dq || !dk || !dv) return ATTN_ERR_NULL_POINTER;
  if (mask_kind < ATTN_MASK_NONE || mask_kind > ATTN_MASK_SLIDING_WINDOW) return ATTN_ERR_MASK;
  if (mask_kind == ATTN_MASK_SLIDING_WINDOW && window < 1) return ATTN_ERR_WINDOW;
  // kept keys (the streaming mask) go with the sliding window
  if (keep_first < 0 || (keep_first > 0 && mask_kind != ATTN_MASK_SLIDING_WINDOW)) return ATTN_ERR_KEEP;
  if ((mask_bits && !aligned(mask_bits, 4)) || (kv_start && !aligned(kv_start, 4)) || (kv_end && !aligned(kv_end, 4)))
    return ATTN_ERR_ALIGNMENT;
  int st = validate(q, k, v, dq, nullptr, N, Hq, H, L, S, E, Ev, scale, mode, sink_logits, nullptr, ATTN_BF16);
  if (st != ATTN_OK) return st;
  if (!aligned(out, 16) || !aligned(dout, 16) || !aligned(lse, 4) || !aligned(dq, 16) || !aligned(dk, 16) ||
      !aligned(dv, 16) || (dsink && !aligned(dsink, 4)))
    return ATTN_ERR_ALIGNMENT;
  int dev = 0, sms = 0, major = 0;
  if (device_info(&dev, &sms, &major) != ATTN_OK) return ATTN_ERR_CUDA;
  if (major != 10) return ATTN_ERR_DEVICE;
  BwdArgs a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.out = out;
  a.dout = dout;
  a.lse = lse;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.dsink = sink_logits ? dsink : nullptr;
  a.sink = sink_logits;
  a.N = N;
  a.Hq = Hq;
  a.H = H;
  a.L = L;
  a.S = S;
  a.E = E;
  a.Ev = Ev;
  a.scale = scale;
  a.rbf = (mode == ATTN_RBF);
  a.mask_kind = keep_first > 0 ? MASK_STREAM : mask_kind;
  a.window = window;
  a.keep = keep_first;
  a.mask_bits = mask_bits;
  a.kv_start = kv_start;
  a.kv_end = kv_end;
  cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
  void* ws = nullptr;
  st = ensure_workspace(dev, bwd_workspace_bytes(a), stream, &ws);
  if (st != ATTN_OK) return st;
  return launch_bwd_bf16(a, ws, stream);
}

int attn_fwd_padded(const void* q, const void* k, const void* v, void* out, float* lse, int N, int Hq, int H, int L,
                    int S, int E, int Ev, float scale, int mode, const float* sink_logits, int mask_kind, int window,
                    const unsigned int* mask_bits, const int* kv_start, const int* kv_end, int dtype,
                    void* stream_ptr) {
  using namespace attn;
  if (mask_kind < ATTN_MASK_NONE || mask_kind > ATTN_MASK_SLIDING_WINDOW) return ATTN_ERR_MASK;
  if (mask_kind == ATTN_MASK_SLIDING_WINDOW && window < 1) return ATTN_ERR_WINDOW;
  if ((mask_bits && !aligned(mask_bits, 4)) || (kv_start && !aligned(kv_start, 4)) || (kv_end && !aligned(kv_end, 4)))
    return ATTN_ERR_ALIGNMENT;
  return forward(q, k, v, out, lse, N, Hq, H, L, S, E, Ev, scale, mode, sink_logits, mask_kind, window, 0, nullptr,
                 dtype, stream_ptr, mask_bits, kv_start, kv_end);
}

int attn_decode_indexed(const void* q, const void* k, const void* v, void* out, float* lse, const int* key_idx,
                        int n_sel, int N, int Hq, int H, int L, int S, int E, int Ev, float scale,
                        const float* sink_logits, int mask_kind, int window, const float* bias, void* stream_ptr) {
  using namespace attn;
  if (!key_idx) return ATTN_ERR_NULL_POINTER;
  if (mask_kind < ATTN_MASK_NONE || mask_kind > ATTN_MASK_SLIDING_WINDOW) return ATTN_ERR_MASK;
  if (mask_kind == ATTN_MASK_SLIDING_WINDOW && window < 1) return ATTN_ERR_WINDOW;
  int st = validate(q, k, v, out, lse, N, Hq, H, L, S, E, Ev, scale, ATTN_DOT, sink_logits, bias, ATTN_BF16);
  if (st != ATTN_OK) return st;
  if (n_sel < 1 || static_cast<long long>(N) * H * n_sel > (1LL << 40)) return ATTN_ERR_BAD_SHAPE;
  if (!aligned(key_idx, 4)) return ATTN_ERR_ALIGNMENT;
  if ((Hq / H) * L > 16) return ATTN_ERR_NOT_DECODE;
  int dev = 0, sms = 0, major = 0;
  if (device_info(&dev, &sms, &major) != ATTN_OK) return ATTN_ERR_CUDA;
  if (major != 10) return ATTN_ERR_DEVICE;
  const AttnArgs a =
      make_args(q, k, v, out, lse, N, Hq, H, L, S, E, Ev, scale, ATTN_DOT, sink_logits, mask_kind, window, 0, bias);
  cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
  void* ws = nullptr;
  const size_t need = decode_gather_workspace_bytes(a, n_sel, sms);
  st = ensure_workspace(dev, need, stream, &ws);
  if (st != ATTN_OK) return st;
  return launch_decode_gather_bf16(a, key_idx, n_sel, ws, need, sms, stream);
}

const char* attn_status_string(int status) {
  switch (status) {
    case ATTN_OK: return "ok";
    case ATTN_ERR_NULL_POINTER: return "a required pointer is NULL";
    case ATTN_ERR_BAD_SHAPE: return "a size is < 1 or too large";
    case ATTN_ERR_GQA: return "Hq is not a multiple of H";
    case ATTN_ERR_HEAD_DIM: return "head dims E and Ev must be 64 or 128";
    case ATTN_ERR_SCALE: return "scale must be finite and > 0";
    case ATTN_ERR_MODE: return "unknown score mode";
    case ATTN_ERR_MASK: return "unknown mask kind";
    case ATTN_ERR_WINDOW: return "sliding window needs window >= 1";
    case ATTN_ERR_KEEP: return "keep_first must be >= 0, and kept keys need the sliding window";
    case ATTN_ERR_SINK: return "ATTN_SINK needs sink logits";
    case ATTN_ERR_DTYPE: return "unknown dtype";
    case ATTN_ERR_ALIGNMENT: return "misaligned pointer (16 bytes for tensors, 4 for lse and sink)";
    case ATTN_ERR_WORKSPACE: return "could not allocate the decode workspace";
    case ATTN_ERR_CUDA: return "CUDA error";
    case ATTN_ERR_DEVICE_TIMEOUT: return "a kernel gave up a bounded wait";
    case ATTN_ERR_DEVICE: return "device is not compute capability 10.x (B200)";
    case ATTN_ERR_SCRATCH_LIMIT: return "the call needs more scratch than the fixed no-allocation area holds";
    case ATTN_ERR_NOT_DECODE: return "not a decode-shaped bf16 call ((Hq/H)*L must be <= 16)";
    default: return "unknown status";
  }
}

void attn_release_workspace(void) {
  using namespace attn;
  std::lock_guard<std::mutex> lock(g_mutex);
  for (int d = 0; d < MAX_DEVICES; ++d) {
    if (!g_ws[d].ptr) continue;
    int cur = 0;
    cudaGetDevice(&cur);
    cudaSetDevice(d);
    cudaDeviceSynchronize();
    cudaFree(g_ws[d].ptr);
    g_ws[d].ptr = nullptr;
    g_ws[d].bytes = 0;
    cudaSetDevice(cur);
  }
}

int attn_device_status(void* stream_ptr) {
  using namespace attn;
  cudaStream_t s = static_cast<cudaStream_t>(stream_ptr);
  const unsigned int a = take_status_prefill(s);
  const unsigned int b = take_status_decode(s);
  const unsigned int c = take_status_bwd(s);
  if (a == 0xFFFFFFFFu || b == 0xFFFFFFFFu || c == 0xFFFFFFFFu) return ATTN_ERR_CUDA;
  return (a | b | c) ? ATTN_ERR_DEVICE_TIMEOUT : ATTN_OK;
}

int attn_version(void) { return 10000; }

int attn_test_wait_timeout(int limit_cycles, void* stream) {
  using namespace attn;
  if (limit_cycles < 1) return ATTN_ERR_BAD_SHAPE;
  int dev = 0, sms = 0, major = 0;
  if (device_info(&dev, &sms, &major) != ATTN_OK) return ATTN_ERR_CUDA;
  if (major != 10) return ATTN_ERR_DEVICE;
  return launch_wait_timeout_test(limit_cycles, static_cast<cudaStream_t>(stream));
}

int attn_test_fail_workspace_allocs(int count) {
  using namespace attn;
  if (count < 0) return ATTN_ERR_BAD_SHAPE;
  std::lock_guard<std::mutex> lock(g_mutex);
  g_fail_allocs = count;
  return ATTN_OK;
}

int attn_exp2_poly_eval(const float* x, float* y, int n, void* stream) {
  if (!x || !y) return ATTN_ERR_NULL_POINTER;
  if (n < 0) return ATTN_ERR_BAD_SHAPE;
  if (n == 0) return ATTN_OK;
  return attn::launch_exp2_poly_eval(x, y, n, static_cast<cudaStream_t>(stream));
}

}  // extern "C"

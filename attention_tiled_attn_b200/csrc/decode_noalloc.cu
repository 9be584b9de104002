// attn_decode_fwd_noalloc: the decode path (key-split partial kernel + combine
// kernel) run on a fixed scratch area that lives in this file instead of the
// library's allocated workspace.
//
// Who needs this: a caller that must not allocate device memory once it is
// running.  Examples are inference services that reserve every byte of GPU
// memory when they start and forbid later allocations so that latency stays
// predictable and an out-of-memory error cannot strike mid-request, and host
// frameworks whose own allocator owns all device memory and does not allow a
// library to allocate behind its back.  Such callers already pass in every
// input and output buffer; this entry point adds no allocation of its own.
//
// The scratch is a file-scope __device__ array of DECODE_SCRATCH_BYTES.  It
// becomes resident on a device when the CUDA runtime loads this library's
// device code into that device's context.  Under the default lazy module
// loading that happens at the first use on the device (here: the first call),
// and it claims the array's 8 MiB plus the code then, so the first call on
// each device belongs in start-up, before the caller reserves the rest of the
// device's memory.  With CUDA_MODULE_LOADING=EAGER the load, and the array,
// come with the context's creation instead.  From then on the array stays
// until the context is destroyed.
//
// Host code cannot pass the array's name to a kernel (on the host that name is
// only a stand-in, not a device address), so the first call in each context
// looks up the array's device address with cudaGetSymbolAddress, with that
// device current, and keeps it with the context's unique id.  A call that
// finds another context current (the old one was destroyed, for instance by
// cudaDeviceReset, and a new one made) looks the address up again.  Make the
// first call on a device before any stream capture is begun.
//
// All calls share the one array, and it keeps whatever the last call left
// there.  Nothing in it needs to start at zero: the partial kernel writes
// every (m, l, acc) slot that the combine kernel of the same call reads.
// Calls that overlap on the GPU (different streams, or different host
// threads without ordering between them) race on the array; order them.

#include <cstdint>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "attn_b200.h"
#include "kernels.h"

namespace {

constexpr size_t DECODE_SCRATCH_BYTES = 8u << 20;  // 8 MiB per device
constexpr int MAX_DEVICES = 64;

static __device__ __align__(256) unsigned char g_decode_scratch[DECODE_SCRATCH_BYTES];

std::mutex g_setup_mutex;
void* g_scratch_addr[MAX_DEVICES] = {nullptr};
unsigned long long g_scratch_ctx[MAX_DEVICES] = {0};  // unique id of the context the address belongs to
int g_scratch_sms[MAX_DEVICES] = {0};
int g_scratch_major[MAX_DEVICES] = {0};

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// The driver's cuCtxGetCurrent / cuCtxGetId, resolved through the runtime (no libcuda link).
bool context_fns(CtxGetCurrentFn* cur, CtxGetIdFn* id) {
  static CtxGetCurrentFn f_cur = nullptr;
  static CtxGetIdFn f_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      f_cur = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      f_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  *cur = f_cur;
  *id = f_id;
  return f_cur != nullptr && f_id != nullptr;
}

// Unique id of the current context, or 0 when none is current yet.
int current_context_id(unsigned long long* id) {
  CtxGetCurrentFn f_cur;
  CtxGetIdFn f_id;
  if (!context_fns(&f_cur, &f_id)) return ATTN_ERR_CUDA;
  CUcontext ctx = nullptr;
  if (f_cur(&ctx) != CUDA_SUCCESS) return ATTN_ERR_CUDA;
  *id = 0;
  if (ctx != nullptr && f_id(ctx, id) != CUDA_SUCCESS) return ATTN_ERR_CUDA;
  return ATTN_OK;
}

// Once per context, with the device current: the scratch array's device
// address in that context and the device's SM count / compute capability.
int setup_device(int dev) {
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  unsigned long long ctx = 0;
  if (current_context_id(&ctx) != ATTN_OK) return ATTN_ERR_CUDA;
  if (g_scratch_addr[dev] != nullptr && ctx != 0 && ctx == g_scratch_ctx[dev]) return ATTN_OK;
  void* ptr = nullptr;
  // creates the device's primary context if none is current yet
  if (cudaGetSymbolAddress(&ptr, g_decode_scratch) != cudaSuccess || ptr == nullptr) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  if (current_context_id(&ctx) != ATTN_OK || ctx == 0) return ATTN_ERR_CUDA;
  int sms = 0, major = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return ATTN_ERR_CUDA;
  g_scratch_sms[dev] = sms;
  g_scratch_major[dev] = major;
  g_scratch_addr[dev] = ptr;
  g_scratch_ctx[dev] = ctx;
  return ATTN_OK;
}

}  // namespace

extern "C" int attn_decode_fwd_noalloc(const void* q, const void* k, const void* v, void* out, float* lse, int N,
                                       int Hq, int H, int L, int S, int E, int Ev, float scale, int mode,
                                       const float* sink_logits, int mask_kind, int window, const float* bias,
                                       void* stream_ptr) {
  if (mask_kind < ATTN_MASK_NONE || mask_kind > ATTN_MASK_SLIDING_WINDOW) return ATTN_ERR_MASK;
  if (mask_kind == ATTN_MASK_SLIDING_WINDOW && window < 1) return ATTN_ERR_WINDOW;
  const int vs = attn::validate(q, k, v, out, lse, N, Hq, H, L, S, E, Ev, scale, mode, sink_logits, bias, ATTN_BF16);
  if (vs != ATTN_OK) return vs;

  attn::AttnArgs a{};
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
  a.bias = bias;
  if (!attn::decode_eligible(a)) return ATTN_ERR_NOT_DECODE;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return ATTN_ERR_CUDA;
  const int st = setup_device(dev);
  if (st != ATTN_OK) return st;
  if (g_scratch_major[dev] != 10) return ATTN_ERR_DEVICE;

  const size_t need = attn::decode_workspace_bytes(a, g_scratch_sms[dev]);
  if (need > DECODE_SCRATCH_BYTES) return ATTN_ERR_SCRATCH_LIMIT;
  return attn::launch_decode_bf16(a, g_scratch_addr[dev], DECODE_SCRATCH_BYTES, g_scratch_sms[dev],
                                  static_cast<cudaStream_t>(stream_ptr));
}

extern "C" size_t attn_decode_noalloc_scratch_bytes(void) { return DECODE_SCRATCH_BYTES; }

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
// The scratch is a file-scope __device__ array of DECODE_SCRATCH_BYTES.
// Every GPU that loads the library holds it until the process exits.  Host
// code cannot pass the array's name to a kernel (on the host that name is only
// a stand-in, not a device address), so the first call on each device looks
// up the array's device address with cudaGetSymbolAddress, with that device
// current, and keeps it for later calls on that device.  Make that first call
// on a device before any stream capture is begun.
//
// All calls share the one array, and it keeps whatever the last call left
// there.  Nothing in it needs to start at zero: the partial kernel writes
// every (m, l, acc) slot that the combine kernel of the same call reads.
// Calls that overlap on the GPU (different streams, or different host
// threads without ordering between them) race on the array; order them.

#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "attn_b200.h"
#include "kernels.h"

namespace {

constexpr size_t DECODE_SCRATCH_BYTES = 8u << 20;  // 8 MiB per device
constexpr int MAX_DEVICES = 64;

static __device__ __align__(256) unsigned char g_decode_scratch[DECODE_SCRATCH_BYTES];

std::mutex g_setup_mutex;
void* g_scratch_addr[MAX_DEVICES] = {nullptr};
int g_scratch_sms[MAX_DEVICES] = {0};
int g_scratch_major[MAX_DEVICES] = {0};

// Once per device, with that device current: the scratch array's device
// address and the device's SM count / compute capability.
int setup_device(int dev) {
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_addr[dev] != nullptr) return ATTN_OK;
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_decode_scratch) != cudaSuccess || ptr == nullptr) {
    cudaGetLastError();
    return ATTN_ERR_CUDA;
  }
  int sms = 0, major = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return ATTN_ERR_CUDA;
  g_scratch_sms[dev] = sms;
  g_scratch_major[dev] = major;
  g_scratch_addr[dev] = ptr;
  return ATTN_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" int attn_decode_fwd_noalloc(const void* q, const void* k, const void* v, void* out, float* lse, int N,
                                       int Hq, int H, int L, int S, int E, int Ev, float scale, int mode,
                                       const float* sink_logits, int mask_kind, int window, const float* bias,
                                       void* stream_ptr) {
  if (!q || !k || !v || !out) return ATTN_ERR_NULL_POINTER;
  if (N < 1 || Hq < 1 || H < 1 || L < 1 || S < 1) return ATTN_ERR_BAD_SHAPE;
  if (Hq % H != 0) return ATTN_ERR_GQA;
  if ((E != 64 && E != 128) || (Ev != 64 && Ev != 128)) return ATTN_ERR_HEAD_DIM;
  if (!(scale > 0.f) || scale > 3.4e38f) return ATTN_ERR_SCALE;
  if (mode < ATTN_DOT || mode > ATTN_SINK) return ATTN_ERR_MODE;
  if (mask_kind < ATTN_MASK_NONE || mask_kind > ATTN_MASK_SLIDING_WINDOW) return ATTN_ERR_MASK;
  if (mask_kind == ATTN_MASK_SLIDING_WINDOW && window < 1) return ATTN_ERR_WINDOW;
  if (mode == ATTN_SINK && sink_logits == nullptr) return ATTN_ERR_SINK;
  const long long NH = static_cast<long long>(N) * H;
  const long long NHq = static_cast<long long>(N) * Hq;
  if (NHq > (1LL << 31) - 1 || NH > (1LL << 31) - 1 || NHq * L > (1LL << 40) || NH * S > (1LL << 40))
    return ATTN_ERR_BAD_SHAPE;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return ATTN_ERR_ALIGNMENT;
  if (bias && !aligned16(bias)) return ATTN_ERR_ALIGNMENT;
  if ((lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) ||
      (sink_logits && (reinterpret_cast<uintptr_t>(sink_logits) & 3u)))
    return ATTN_ERR_ALIGNMENT;

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

// Internal launch interface shared by the C-ABI layer and the kernel files.
#pragma once

#include <cstddef>
#include <cuda_runtime.h>

namespace attn {

// MASK_STREAM: the sliding window plus the first `keep` keys, which stay visible
// to every query at or after them (StreamingLLM's kept initial tokens).
enum MaskKind { MASK_NONE = 0, MASK_CAUSAL = 1, MASK_WINDOW = 2, MASK_STREAM = 3 };

// Validated arguments of one forward call (see include/attn_b200.h).
struct AttnArgs {
  const void* q;
  const void* k;
  const void* v;
  void* out;
  float* lse;          // nullable
  int N, Hq, H, L, S, E, Ev;
  float scale;
  bool rbf;
  const float* sink;   // [Hq] or nullptr
  int mask_kind;
  int window;
  const float* bias;   // [L, S] or nullptr
  int keep;            // MASK_STREAM: number of initial keys always visible (0 otherwise)
  const uint32_t* mask_bits;  // [L][ceil(S/32)] keep bits (bit j%32 of word j/32), or nullptr
  const int* kv_start;        // [N] first non-padding key per batch, or nullptr (0)
  const int* kv_end;          // [N] one past the last non-padding key per batch, or nullptr (S)
};

constexpr float LOG2E = 1.4426950408889634f;
constexpr float LN2 = 0.6931471805599453f;

// Checks shared by every forward entry point once it has checked its own mask
// arguments (defined in attn_abi.cu); returns ATTN_OK or a negative status.
int validate(const void* q, const void* k, const void* v, void* out, float* lse, int N, int Hq, int H, int L, int S,
             int E, int Ev, float scale, int mode, const float* sink_logits, const float* bias, int dtype);

// Each launcher returns 0 or a negative attn_status code.
// bf16 prefill.  A float bias (outside the streaming mask) is first turned into keep
// bits in `ws` (prefill_workspace_bytes(a) bytes, 0 when none is needed).
size_t prefill_workspace_bytes(const AttnArgs& a);
int launch_prefill_bf16(const AttnArgs& a, void* ws, size_t ws_bytes, cudaStream_t stream);
int launch_fp32(const AttnArgs& a, cudaStream_t stream);

// Decode (bf16, (Hq/H) * L <= 16): key-split partial kernel + combine kernel.
bool decode_eligible(const AttnArgs& a);
size_t decode_workspace_bytes(const AttnArgs& a, int num_sms);
// Decode over listed keys: key_idx [N*H][n_sel] device array of key positions
// (entries outside [0, S) select nothing); same workspace scheme.
size_t decode_gather_workspace_bytes(const AttnArgs& a, int n_sel, int num_sms);
int launch_decode_gather_bf16(const AttnArgs& a, const int* key_idx, int n_sel, void* workspace,
                              size_t workspace_bytes, int num_sms, cudaStream_t stream);
int launch_decode_bf16(const AttnArgs& a, void* workspace, size_t workspace_bytes, int num_sms,
                       cudaStream_t stream);

// Resolves cuTensorMapEncodeTiled through the runtime (no libcuda link).
void* tensor_map_encoder();

// bf16 [heads, rows, dim] tensor map with a 64 x box_rows x 1 box, 128-byte
// swizzle and zero fill outside the tensor (defined in attn_abi.cu).
bool make_map_rows(void* map, const void* base, int dim, long long rows, long long heads, int box_rows);

// The prefill softmax's software base-2 exponential applied to n floats (verification).
int launch_exp2_poly_eval(const float* x, float* y, int n, cudaStream_t stream);

// Read-and-clear of each kernel file's device fault word (synchronises `s`).
// Backward (bf16): validated arguments of one attn_bwd call.
struct BwdArgs {
  const void* q;       // [N, Hq, L, E] bf16
  const void* k;       // [N, H, S, E]
  const void* v;       // [N, H, S, Ev]
  const void* out;     // [N, Hq, L, Ev] forward output
  const void* dout;    // [N, Hq, L, Ev] gradient of the loss with respect to out
  const float* lse;    // [N, Hq, L] forward lse (natural log, sink included)
  float* dq;           // [N, Hq, L, E]
  float* dk;           // [N, H, S, E]
  float* dv;           // [N, H, S, Ev]
  float* dsink;        // [Hq] or nullptr
  const float* sink;   // [Hq] or nullptr
  int N, Hq, H, L, S, E, Ev;
  float scale;
  bool rbf;
  int mask_kind, window;
  int keep;                   // MASK_STREAM: kept initial keys
  const uint32_t* mask_bits;  // [L][ceil(S/32)] keep bits, or nullptr
  const int* kv_start;        // [N] or nullptr
  const int* kv_end;          // [N] or nullptr
};
size_t bwd_workspace_bytes(const BwdArgs& a);
int launch_bwd_bf16(const BwdArgs& a, void* workspace, cudaStream_t stream);
unsigned int take_status_bwd(cudaStream_t s);

unsigned int take_status_prefill(cudaStream_t s);
// A kernel whose one bounded wait runs out after limit_cycles (failure-path check).
int launch_wait_timeout_test(int limit_cycles, cudaStream_t stream);
unsigned int take_status_decode(cudaStream_t s);

}  // namespace attn

// fp32 fused attention forward on the FFMA pipe.
//
// For float32 inputs the tensor cores (TF32) would round q and k to 10-bit
// mantissas, far outside the 1e-5 agreement an fp32 result should reach, so
// this path keeps every product and sum in IEEE fp32: a tiled online-softmax
// loop (64 query rows x 64 keys per step, 128 threads, each thread a 4 x 8
// block of logits and a 4 x Ev/8 block of the output), natural-base expf.
// It covers every score mode, mask kind, bias, sink and GQA setting.
//
// Method: page "어텐션 메커니즘" §6 (tiling with an online softmax, exact);
// page "Dot-Product Attention을 거리 기반 RBF-Attention으로 교체한 실험기"
// (RBF as a dot product with a key-norm penalty formed from the key tile);
// page "Attention Sink" §4.2 (sink in the denominator only).

#include <cstdint>
#include <cuda_runtime.h>

#include "kernels.h"

namespace attn {

namespace {

constexpr int FBM = 64;
constexpr int FBN = 64;
constexpr int FTHREADS = 128;

struct F32Params {
  const float* q;
  const float* k;
  const float* v;
  float* out;
  float* lse;
  const float* sink;
  const float* bias;
  int N, Hq, H, L, S, group;
  int mask_kind, window, keep;
  float scale;
  const uint32_t* mask_bits;  // [L][mask_words] keep bits or nullptr
  const int* kv_start;        // [N] or nullptr
  const int* kv_end;          // [N] or nullptr
  int mask_words;
};

template <int E, int EV>
struct F32Smem {
  float q[FBM][E + 1];
  float k[FBN][E + 1];
  float v[FBN][EV];
  float p[FBM][FBN + 1];
  float kn[FBN];
};

template <int E, int EV, bool RBF>
__global__ void __launch_bounds__(FTHREADS) fp32_attn_kernel(const F32Params p) {
  extern __shared__ float4 smem_f4[];
  auto& sm = *reinterpret_cast<F32Smem<E, EV>*>(smem_f4);
  const int tid = threadIdx.x;
  const int rg = tid >> 3;  // row group: rows rg*4 .. rg*4+3
  const int cg = tid & 7;   // column group: columns cg + 8*c

  const int n_rb = (p.L + FBM - 1) / FBM;
  const int rb = n_rb - 1 - blockIdx.x;  // heavy (late) row blocks first
  const int nh = blockIdx.y;
  const int n = nh / p.Hq;
  const int hq = nh % p.Hq;
  const int kvh = hq / p.group;
  const int r0 = rb * FBM;

  const float* qg = p.q + ((size_t)nh * p.L) * E;
  const float* kg = p.k + ((size_t)(n * p.H + kvh) * p.S) * E;
  const float* vg = p.v + ((size_t)(n * p.H + kvh) * p.S) * EV;

  // query tile
  for (int x = tid; x < FBM * E / 4; x += FTHREADS) {
    const int r = x / (E / 4), c4 = x % (E / 4);
    float4 val = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r0 + r < p.L) val = reinterpret_cast<const float4*>(qg + (size_t)(r0 + r) * E)[c4];
    sm.q[r][4 * c4 + 0] = val.x;
    sm.q[r][4 * c4 + 1] = val.y;
    sm.q[r][4 * c4 + 2] = val.z;
    sm.q[r][4 * c4 + 3] = val.w;
  }

  // key range of the row block
  const int off = p.S - p.L;
  const int r_last = min(r0 + FBM - 1, p.L - 1);
  const bool windowed = p.mask_kind == MASK_WINDOW || p.mask_kind == MASK_STREAM;
  const int hi_blk = (p.mask_kind == MASK_NONE) ? p.S : min(p.S, r_last + off + 1);
  const int lo_blk = (windowed && p.keep == 0) ? max(0, r0 + off - p.window + 1) : 0;
  // key padding of this batch: keys outside [ks, ke) are never visible
  const int ks = p.kv_start ? max(0, p.kv_start[n]) : 0;
  const int ke = p.kv_end ? min(p.S, p.kv_end[n]) : p.S;
  const int jb_lo = max(lo_blk, ks) / FBN;
  const int jb_hi = min(hi_blk, ke) > max(lo_blk, ks) ? (min(hi_blk, ke) + FBN - 1) / FBN : jb_lo;
  // streaming: key blocks between the kept head and the first row's window are invisible to all rows
  const int gap_lo = (p.keep + FBN - 1) / FBN;
  const int gap_hi = (p.mask_kind == MASK_STREAM) ? max(0, r0 + off - p.window + 1) / FBN : 0;

  // key j visible to row i iff j < hi_i and (j >= lo_i or j < keep)
  int lo_i[4], hi_i[4];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int i = r0 + rg * 4 + r;
    lo_i[r] = windowed ? i + off - p.window + 1 : 0;
    hi_i[r] = (p.mask_kind == MASK_NONE) ? p.S : min(p.S, i + off + 1);
  }

  float m_run[4], l_run[4], acc[4][EV / 8];
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    m_run[r] = -INFINITY;
    l_run[r] = 0.f;
#pragma unroll
    for (int c = 0; c < EV / 8; ++c) acc[r][c] = 0.f;
  }

  for (int jb = jb_lo; jb < jb_hi; ++jb) {
    if (jb >= gap_lo && jb < gap_hi) continue;
    const int k0 = jb * FBN;
    __syncthreads();
    for (int x = tid; x < FBN * E / 4; x += FTHREADS) {
      const int r = x / (E / 4), c4 = x % (E / 4);
      float4 val = make_float4(0.f, 0.f, 0.f, 0.f);
      if (k0 + r < p.S) val = reinterpret_cast<const float4*>(kg + (size_t)(k0 + r) * E)[c4];
      sm.k[r][4 * c4 + 0] = val.x;
      sm.k[r][4 * c4 + 1] = val.y;
      sm.k[r][4 * c4 + 2] = val.z;
      sm.k[r][4 * c4 + 3] = val.w;
    }
    for (int x = tid; x < FBN * EV / 4; x += FTHREADS) {
      const int r = x / (EV / 4), c4 = x % (EV / 4);
      float4 val = make_float4(0.f, 0.f, 0.f, 0.f);
      if (k0 + r < p.S) val = reinterpret_cast<const float4*>(vg + (size_t)(k0 + r) * EV)[c4];
      reinterpret_cast<float4*>(&sm.v[r][0])[c4] = val;
    }
    __syncthreads();
    if (RBF) {
      if (tid < FBN) {
        float s = 0.f;
#pragma unroll 8
        for (int d = 0; d < E; ++d) s = fmaf(sm.k[tid][d], sm.k[tid][d], s);
        sm.kn[tid] = s;
      }
      __syncthreads();
    }

    float z[4][8];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int c = 0; c < 8; ++c) z[r][c] = 0.f;
#pragma unroll 4
    for (int d = 0; d < E; ++d) {
      float a[4], b[8];
#pragma unroll
      for (int r = 0; r < 4; ++r) a[r] = sm.q[rg * 4 + r][d];
#pragma unroll
      for (int c = 0; c < 8; ++c) b[c] = sm.k[cg + 8 * c][d];
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 8; ++c) z[r][c] = fmaf(a[r], b[c], z[r][c]);
    }

#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int i = r0 + rg * 4 + r;
      float mt = -INFINITY;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const int key = k0 + cg + 8 * c;
        float zz = RBF ? (2.f * p.scale) * z[r][c] - p.scale * sm.kn[cg + 8 * c] : p.scale * z[r][c];
        if (key >= hi_i[r] || (key < lo_i[r] && key >= p.keep)) zz = -INFINITY;
        if (key < ks || key >= ke) zz = -INFINITY;
        if (p.mask_bits != nullptr && i < p.L && key < p.S &&
            !((p.mask_bits[(size_t)i * p.mask_words + (key >> 5)] >> (key & 31)) & 1u))
          zz = -INFINITY;
        if (p.bias != nullptr && i < p.L && key < p.S) zz += p.bias[(size_t)i * p.S + key];
        z[r][c] = zz;
        mt = fmaxf(mt, zz);
      }
      mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 1));
      mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 2));
      mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 4));
      const float m_new = fmaxf(m_run[r], mt);
      const float mu = (m_new == -INFINITY) ? 0.f : m_new;
      const float alpha = (m_run[r] == -INFINITY) ? 0.f : expf(m_run[r] - mu);
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const float pv = expf(z[r][c] - mu);
        sm.p[rg * 4 + r][cg + 8 * c] = pv;
        rs += pv;
      }
      rs += __shfl_xor_sync(0xffffffffu, rs, 1);
      rs += __shfl_xor_sync(0xffffffffu, rs, 2);
      rs += __shfl_xor_sync(0xffffffffu, rs, 4);
      l_run[r] = l_run[r] * alpha + rs;
      m_run[r] = m_new;
#pragma unroll
      for (int c = 0; c < EV / 8; ++c) acc[r][c] *= alpha;
    }
    __syncthreads();
#pragma unroll 4
    for (int j = 0; j < FBN; ++j) {
      float pr[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) pr[r] = sm.p[rg * 4 + r][j];
#pragma unroll
      for (int c = 0; c < EV / 8; ++c) {
        const float vv = sm.v[j][cg + 8 * c];
#pragma unroll
        for (int r = 0; r < 4; ++r) acc[r][c] = fmaf(pr[r], vv, acc[r][c]);
      }
    }
  }

  // epilogue: sink in the denominator only
  const float s = p.sink ? p.sink[hq] : -INFINITY;
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int i = r0 + rg * 4 + r;
    if (i >= p.L) continue;
    const float M = fmaxf(m_run[r], s);
    float inv = 0.f, lse = -INFINITY;
    if (M != -INFINITY) {
      const float a = (m_run[r] == -INFINITY) ? 0.f : expf(m_run[r] - M);
      const float d = l_run[r] * a + ((s == -INFINITY) ? 0.f : expf(s - M));
      if (d > 0.f) {
        inv = a / d;
        lse = M + logf(d);
      }
    }
    float* orow = p.out + ((size_t)nh * p.L + i) * EV;
#pragma unroll
    for (int c = 0; c < EV / 8; ++c) orow[cg + 8 * c] = acc[r][c] * inv;
    if (p.lse && cg == 0) p.lse[(size_t)nh * p.L + i] = lse;
  }
}

template <int E, int EV, bool RBF>
int launch_f32_impl(const AttnArgs& a, cudaStream_t stream) {
  F32Params p{};
  p.q = static_cast<const float*>(a.q);
  p.k = static_cast<const float*>(a.k);
  p.v = static_cast<const float*>(a.v);
  p.out = static_cast<float*>(a.out);
  p.lse = a.lse;
  p.sink = a.sink;
  p.bias = a.bias;
  p.N = a.N;
  p.Hq = a.Hq;
  p.H = a.H;
  p.L = a.L;
  p.S = a.S;
  p.group = a.Hq / a.H;
  p.mask_kind = a.mask_kind;
  p.window = a.window;
  p.keep = a.keep;
  p.scale = a.scale;
  p.mask_bits = a.mask_bits;
  p.kv_start = a.kv_start;
  p.kv_end = a.kv_end;
  p.mask_words = (a.S + 31) / 32;
  const int smem = sizeof(F32Smem<E, EV>);
  auto kern = fp32_attn_kernel<E, EV, RBF>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) return -13;
  dim3 grid((a.L + FBM - 1) / FBM, a.N * a.Hq);
  kern<<<grid, FTHREADS, smem, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? 0 : -13;
}

}  // namespace

int launch_fp32(const AttnArgs& a, cudaStream_t stream) {
  const bool r = a.rbf;
#define ATTN_F32_CASE(e, ev)                                                   \
  if (a.E == e && a.Ev == ev) return r ? launch_f32_impl<e, ev, true>(a, stream) \
                                       : launch_f32_impl<e, ev, false>(a, stream);
  ATTN_F32_CASE(64, 64)
  ATTN_F32_CASE(128, 128)
  ATTN_F32_CASE(64, 128)
  ATTN_F32_CASE(128, 64)
#undef ATTN_F32_CASE
  return -4;
}

}  // namespace attn

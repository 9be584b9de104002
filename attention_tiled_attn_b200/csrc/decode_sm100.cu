// bf16 attention forward for short query blocks (decode): split over keys.
//
// With L = 1 the whole batch holds only N*H independent (batch, KV head)
// units of (Hq/H)*L query rows each, far too few to fill 148 SMs, and every
// key/value byte is read exactly once, so the pass is bound by HBM bandwidth.
// The key axis of every unit is cut into 64-key chunks and the N*H*chunks
// work list is split evenly across a persistent grid (one CTA per SM): CTA b
// takes chunks [b*T/G, (b+1)*T/G), which may span the end of one unit and the
// start of the next.  For each unit segment it writes a partial
// (m, l, acc[Ev]) per query row into slot b + u (CTA b, unit u: the pairs are
// distinct and each unit's slots are consecutive) and counts it in a per-unit
// arrival counter; the CTA whose count completes the unit merges all of the
// unit's partials (one warp per query row) and adds the sink logit (page
// "Attention Sink" §4.2: the sink joins the denominator only).  The counters are
// zeroed before each launch; there is no second kernel.
//
// RBF variant: the score is -scale ||q - k||^2 in the expanded frame
// 2 scale q.k - scale ||k||^2 (page "Dot-Product Attention을 거리 기반
// RBF-Attention으로 교체한 실험기", 섹션별 상세); each consumer warp computes
// ||k||^2 of its 16 keys from the staged K chunk.
//
// Per CTA: one TMA producer warp streams K and V chunks (3-D tensor maps,
// 128-byte swizzle, zero fill past S) through a ring of stages; two groups of
// four consumer warps take alternate chunks (one group in the listed-key variant),
// each warp 16 keys of its group's chunks.  The query rows of a unit (the
// Hq/H heads of the KV group times L positions, at most 16) form the M = 16
// side of mma.sync m16n8k16 products: S = Q K^T, then O += P V with P kept
// in registers.  Each warp keeps its own online-softmax state; the states are
// merged through shared memory at the end of a segment.
//
// Masks follow the bottom-right alignment of page "SDPA란 무엇인가" §4
// (trap 3): query i of L sits at key position i + S - L.
//
// GATHER variant: exact attention over a listed key subset (page "기술 요약:
// SOCKET - 희소 어텐션을 위한 SOft Collision Kernel EsTimator", 방법론, step 4:
// top-k keys are selected, then exact attention runs on them).  A unit's chunks
// are 64 consecutive list entries; the producer warp gathers the listed K and
// V rows with 16-byte cp.async copies (two whole 256-byte rows per warp
// instruction at E = 128, four warps) into the same swizzled stage layout, and stores the
// chunk's key positions in shared memory for the consumers' masks.  The list
// entries are loaded two chunks ahead.  (One bulk copy per row through the TMA
// engine measured half the throughput: at 256 bytes its per-copy cost dominates.)

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kernels.h"
#include "ptx_sm100.cuh"

namespace attn {

namespace {

constexpr int DC = 64;             // keys per chunk
constexpr int DWARPS = 4;          // consumer warps per group (16 keys of a chunk each)
// Consumer groups: two groups of four warps take alternate chunks, so each SMSP runs two
// consumer warps and one's dependency chains hide behind the other's (the listed-key
// variant, with its four gathering warps, keeps one group).
template <bool GATHER>
__host__ __device__ constexpr int n_groups() { return GATHER ? 1 : 2; }
constexpr int DTHREADS = (2 * DWARPS + 1) * 32;  // two consumer groups + the producer
// GATHER: producer warps, each issuing every GWARPS-th copy instruction of a chunk.  One warp
// keeps too few copies in flight for random rows; 4 measured best (5 and 6 were slower).
constexpr int GWARPS = 4;
constexpr float D_RESCALE_THRESHOLD = 8.0f;

struct DecodeParams {  // 128 bytes: kept at that size, the kernels' code generation depends on it
  const __nv_bfloat16* q;
  __nv_bfloat16* out;
  float* lse;
  const float* sink;
  const float* bias;
  float* ws_acc;    // [slots][16][Ev]
  float* ws_ml;     // [slots][16][2]
  long long T;      // total chunks = N*H*nc
  int N, Hq, H, L, S, group, R;
  int mask_kind, window;
  int kb_win;       // first chunk after the head part (the window's; the first visible one otherwise)
  int nc;           // chunks per unit (head part + window part)
  int G;            // persistent CTAs
  int n_units;      // N * H
  float c_dot;      // scale * log2e
  int keep;         // streaming mask: initial keys every later query sees
  int nc_head;      // streaming mask: chunks of the kept initial keys (0 otherwise)
};
static_assert(sizeof(DecodeParams) == 128, "DecodeParams layout");

// GATHER and EXT only (a separate kernel argument, so the other variants'
// parameter block stays as it is)
struct ExtraArgs {
  const int* idx;            // GATHER: [N*H][n_sel] key positions
  const __nv_bfloat16* k;    // GATHER: [N*H][S][E]
  const __nv_bfloat16* v;    // GATHER: [N*H][S][Ev]
  int n_sel;
  const uint32_t* bits;      // EXT: [L][words] keep bits (bit j % 32 of word j / 32), or nullptr
  const int* kv_start;       // EXT: [N] first non-padding key, or nullptr
  const int* kv_end;         // EXT: [N] one past the last non-padding key, or nullptr
  int words;                 // EXT: ceil(S / 32)
};

template <int E, int EV, bool GATHER = false>
struct DCfg {
  static constexpr int K_BYTES = DC * E * 2;  // V part of a stage starts here
  static constexpr int STAGE_BYTES = DC * (E + EV) * 2;
  // With two consumer groups taking alternate chunks the count is even, so stage s is
  // always consumed by group s % 2: each full barrier then has one waiting group, which
  // waits its phases in order (a group that waited on a stage shared with the other could
  // ask for the phase after an incomplete one, and its parity test would pass early).
  static constexpr int NSTAGE = (E + EV >= 256) ? (GATHER ? 5 : 6) : (GATHER ? 7 : 8);
  static_assert(GATHER || NSTAGE % 2 == 0, "each stage belongs to one consumer group");
  static constexpr int OFF_STAGES = 0;
  static constexpr int OFF_MERGE = NSTAGE * STAGE_BYTES;              // [DWARPS][16][EV] f32
  static constexpr int OFF_ML = OFF_MERGE + DWARPS * 16 * EV * 4;     // [DWARPS][16][2] f32
  static constexpr int OFF_BAR = OFF_ML + DWARPS * 16 * 2 * 4;
  static constexpr int OFF_MISC = OFF_BAR + 2 * NSTAGE * 8;
  static constexpr int OFF_KEYS = OFF_MISC + 16;                      // [NSTAGE][DC] int (GATHER)
  static constexpr int SMEM_BYTES = OFF_KEYS + (GATHER ? NSTAGE * DC * 4 : 0) + 1024;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

__device__ __forceinline__ long long seg_start(long long b, long long T, int G) { return (b * T) / G; }
// The CTA whose chunk range [seg_start(b), seg_start(b + 1)) holds chunk c.
__device__ __forceinline__ long long cta_of(long long c, long long T, int G) { return ((c + 1) * G - 1) / T; }

// First key of a unit's local chunk.  STREAM (the streaming mask with kept keys,
// a compile-time switch): the head part, then the window part.
template <bool STREAM>
__device__ __forceinline__ int chunk_key0(const DecodeParams& p, int local) {
  if constexpr (STREAM) return (local < p.nc_head ? local : p.kb_win + (local - p.nc_head)) * DC;
  return (p.kb_win + local) * DC;
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// 16-byte global -> shared copy through L2 only
// 16-byte global -> shared copy through L2 only
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
// arrive on an mbarrier once this thread's earlier cp.async copies have landed;
// the arrival counts toward the barrier's expected count
__device__ __forceinline__ void cp_async_mbar_arrive(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// every consumer warp (named barrier 1); the _and form returns the AND of the threads' flags
template <int NT>
__device__ __forceinline__ void consumer_bar() { asm volatile("bar.sync 1, %0;" ::"n"(NT) : "memory"); }
template <int NT>
__device__ __forceinline__ bool consumer_bar_and(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.and.pred p, 1, %2, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "n"(NT)
      : "memory");
  return r != 0;
}

// byte offset of (row, 16-byte chunk c) inside a swizzled chunk buffer of 64-row, 128-byte boxes
__device__ __forceinline__ uint32_t sw_off(int row, int c16) {
  return (c16 >> 3) * (DC * 128) + row * 128 + (((c16 & 7) ^ (row & 7)) << 4);
}

// The merge of one unit's partials for query row r, by one warp, 32 segments at a
// time: lane j reads segment j's (m, l), shuffles reduce the block's maximum and
// denominator, and each lane accumulates EV/32 output columns over the block's
// segments with vector loads.  The sink joins the denominator only.  The partials
// were written by other CTAs: they are read through L2 (ld.global.cg).
template <int EV>
__device__ __forceinline__ void combine_row(const DecodeParams& p, long long u, int r, int lane) {
  constexpr int PER = EV / 32;  // output columns per lane
  const int n = static_cast<int>(u / p.H), kvh = static_cast<int>(u % p.H);
  const long long b0 = cta_of(u * p.nc, p.T, p.G), b1 = cta_of(u * p.nc + p.nc - 1, p.T, p.G);
  const int nseg = static_cast<int>(b1 - b0 + 1);
  const size_t slot0 = static_cast<size_t>(b0 + u);  // the unit's segments: slots slot0 .. slot0 + nseg - 1
  const int hq = kvh * p.group + r / p.L;
  const int i = r % p.L;
  const float s2 = p.sink ? p.sink[hq] * LOG2E : -INFINITY;
  float M = s2, l = 0.f;
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  for (int k0 = 0; k0 < nseg; k0 += 32) {
    // lane j holds segment k0 + j's (m, l); the block's maximum rescales what came before
    float2 ml = make_float2(-INFINITY, 0.f);
    if (k0 + lane < nseg) ml = __ldcg(reinterpret_cast<const float2*>(p.ws_ml + ((slot0 + k0 + lane) * 16 + r) * 2));
    float bm = ml.x;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, o));
    const float Mn = fmaxf(M, bm);
    if (Mn == -INFINITY) continue;
    if (Mn > M) {
      const float sc = ex2(M - Mn);  // 0 while M is -inf
      l *= sc;
#pragma unroll
      for (int e = 0; e < PER; ++e) acc[e] *= sc;
      M = Mn;
    }
    const float a = ml.x == -INFINITY ? 0.f : ex2(ml.x - M);
    float la = a * ml.y;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) la += __shfl_xor_sync(0xffffffffu, la, o);
    l += la;
    const int cnt = min(32, nseg - k0);
#pragma unroll 8
    for (int j = 0; j < cnt; ++j) {
      const float aj = __shfl_sync(0xffffffffu, a, j);
      const float* src = p.ws_acc + ((slot0 + k0 + j) * 16 + r) * EV + lane * PER;
      if constexpr (PER == 4) {
        const float4 v = __ldcg(reinterpret_cast<const float4*>(src));
        acc[0] = fmaf(aj, v.x, acc[0]);
        acc[1] = fmaf(aj, v.y, acc[1]);
        acc[2] = fmaf(aj, v.z, acc[2]);
        acc[3] = fmaf(aj, v.w, acc[3]);
      } else {
        const float2 v = __ldcg(reinterpret_cast<const float2*>(src));
        acc[0] = fmaf(aj, v.x, acc[0]);
        acc[1] = fmaf(aj, v.y, acc[1]);
      }
    }
  }
  if (M != -INFINITY) l += ex2(s2 - M);
  const float inv = (l > 0.f) ? 1.f / l : 0.f;
  const size_t orow = (static_cast<size_t>(n) * p.Hq + hq) * p.L + i;
  __nv_bfloat16* op = p.out + orow * EV + lane * PER;
#pragma unroll
  for (int e = 0; e < PER; e += 2)
    *reinterpret_cast<uint32_t*>(op + e) = pack_bf16x2(acc[e] * inv, acc[e + 1] * inv);
  if (lane == 0 && p.lse) p.lse[orow] = (l > 0.f) ? (M + __log2f(l)) * LN2 : -INFINITY;
}

template <int E, int EV, bool STREAM, bool GATHER, bool EXT, bool RBF>
// 288 threads (256 for the listed-key variant): nine warps put three on one SMSP, whose
// quarter of the register file (16384) caps a thread at 168 registers
__global__ void __launch_bounds__(GATHER ? (DWARPS + GWARPS) * 32 : DTHREADS, 1)
    decode_partial_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                          const DecodeParams p, const ExtraArgs ga) {
  using C = DCfg<E, EV, GATHER>;
  static_assert(!(GATHER && RBF), "listed-key decode takes the dot score");
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t sb = (raw_addr + 1023u) & ~1023u;
  uint8_t* sp = smem_raw + (sb - raw_addr);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sp + C::OFF_MISC);
  volatile int* last_flag = reinterpret_cast<volatile int*>(sp + C::OFF_MISC + 4);  // fused combine
  auto full_bar = [&](int s) -> uint32_t { return sb + C::OFF_BAR + 8u * s; };
  auto empty_bar = [&](int s) -> uint32_t { return sb + C::OFF_BAR + 8u * (C::NSTAGE + s); };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const long long c_begin = seg_start(blockIdx.x, p.T, p.G);
  const long long c_end = seg_start(blockIdx.x + 1, p.T, p.G);

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    for (int s = 0; s < C::NSTAGE; ++s) {
      // GATHER: each producer lane arrives twice, once when its copies land and once for its key positions
      mbar_init(full_bar(s), GATHER ? 64 * GWARPS : 1);
      mbar_init(empty_bar(s), DWARPS);
    }
    fence_barrier_init();
  }
  __syncthreads();
  if (c_end <= c_begin) return;

  if (GATHER && warp >= DWARPS) {
    const int pw = warp - DWARPS;  // this warp issues copy instructions pw, pw + GWARPS, ...
    // ---------------- gathering producer (whole warp) ----------------
    int* keys_s = reinterpret_cast<int*>(sp + C::OFF_KEYS);
    // the list entries of chunk c: lane l holds entries l and l + 32 (-1 past the list's end);
    // they are loaded two chunks ahead so their latency overlaps earlier chunks' copies
    auto load_list = [&](long long c, int& a, int& b) {
      const long long u = c / p.nc;
      const int local = static_cast<int>(c % p.nc);
      const int* lst = ga.idx + static_cast<size_t>(u) * ga.n_sel + static_cast<size_t>(local) * DC;
      const int n_here = min(DC, ga.n_sel - local * DC);
      a = lane < n_here ? __ldg(lst + lane) : -1;
      b = lane + 32 < n_here ? __ldg(lst + lane + 32) : -1;
    };
    constexpr int PK = E / 8, RK = 32 / PK;  // 16-byte pieces per K row, K rows per warp instruction
    constexpr int PV = EV / 8, RV = 32 / PV;
    int na0 = -1, na1 = -1, nb0 = -1, nb1 = -1;  // chunks c + 1 and c + 2
    if (c_begin < c_end) load_list(c_begin, na0, na1);
    if (c_begin + 1 < c_end) load_list(c_begin + 1, nb0, nb1);
    for (long long c = c_begin; c < c_end; ++c) {
      const int idx = static_cast<int>(c - c_begin);
      const int s = idx % C::NSTAGE;
      const uint32_t ph = (idx / C::NSTAGE) & 1;
      int j0 = na0, j1 = na1;
      na0 = nb0;
      na1 = nb1;
      if (c + 2 < c_end) load_list(c + 2, nb0, nb1);
      const bool w_ok = mbar_wait(empty_bar(s), ph ^ 1);
      if (!__all_sync(0xffffffffu, w_ok) || *abort_flag) {
        if (lane == 0) *abort_flag = 1;
        break;
      }
      const long long u = c / p.nc;
      j0 = (j0 >= 0 && j0 < p.S) ? j0 : -1;  // entries outside [0, S) select nothing
      j1 = (j1 >= 0 && j1 < p.S) ? j1 : -1;
      if (pw == 0) {
        keys_s[s * DC + lane] = j0;
        keys_s[s * DC + 32 + lane] = j1;
      }
      const __nv_bfloat16* kb = ga.k + static_cast<size_t>(u) * p.S * E;
      const __nv_bfloat16* vb = ga.v + static_cast<size_t>(u) * p.S * EV;
      const uint32_t kdst = sb + C::OFF_STAGES + s * C::STAGE_BYTES;
      const uint32_t vdst = kdst + C::K_BYTES;
      // rows without a key (padding) copy row 0 of the unit; the consumers mask them
#pragma unroll 4
      for (int m = pw; m < DC / RK; m += GWARPS) {
        const int r = m * RK + lane / PK;  // rows of one instruction are all below 32 or all above
        const int jr = __shfl_sync(0xffffffffu, m * RK < 32 ? j0 : j1, r & 31);
        const int col = lane % PK;
        cp_async16(kdst + sw_off(r, col), kb + static_cast<size_t>(jr < 0 ? 0 : jr) * E + col * 8);
      }
#pragma unroll 4
      for (int m = pw; m < DC / RV; m += GWARPS) {
        const int r = m * RV + lane / PV;
        const int jr = __shfl_sync(0xffffffffu, m * RV < 32 ? j0 : j1, r & 31);
        const int col = lane % PV;
        cp_async16(vdst + sw_off(r, col), vb + static_cast<size_t>(jr < 0 ? 0 : jr) * EV + col * 8);
      }
      cp_async_mbar_arrive(full_bar(s));
      mbar_arrive(full_bar(s));  // releases this lane's key positions
    }
    cp_async_wait_all();  // no copy may still be in flight at exit
    return;
  }
  constexpr int NGRP = n_groups<GATHER>();
  constexpr int NCW = NGRP * DWARPS;  // consumer warps
  constexpr int NCT = NCW * 32;       // consumer threads
  if (warp == NCW) {
    // ---------------- producer ----------------
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      int issued = 0;
      for (long long c = c_begin; c < c_end; ++c) {
        const int idx = static_cast<int>(c - c_begin);
        const int s = idx % C::NSTAGE;
        const uint32_t ph = (idx / C::NSTAGE) & 1;
        bool ok = mbar_wait(empty_bar(s), ph ^ 1);
        if (!ok || *abort_flag) {
          *abort_flag = 1;
          break;
        }
        const long long u = c / p.nc;
        const int key0 = chunk_key0<STREAM>(p, static_cast<int>(c % p.nc));
        const uint32_t dst = sb + C::OFF_STAGES + s * C::STAGE_BYTES;
        mbar_arrive_expect_tx(full_bar(s), C::STAGE_BYTES);
        for (int b = 0; b < E / 64; ++b)
          tma_load_3d(dst + b * (DC * 128), &tm_k, full_bar(s), b * 64, key0, static_cast<int>(u));
        for (int b = 0; b < EV / 64; ++b)
          tma_load_3d(dst + E * DC * 2 + b * (DC * 128), &tm_v, full_bar(s), b * 64, key0, static_cast<int>(u));
        issued = idx + 1;
      }
      // drain: the last NSTAGE copies (one per stage) have landed before exit
      for (int idx = issued > C::NSTAGE ? issued - C::NSTAGE : 0; idx < issued; ++idx)
        mbar_wait(full_bar(idx % C::NSTAGE), (idx / C::NSTAGE) & 1);
    }
    return;
  }

  // ---------------- consumers ----------------
  const int grp = warp / DWARPS;  // consumer group: the chunks idx = c - c_begin with idx % NGRP == grp
  const int wq = warp % DWARPS;   // this warp's 16 keys of each chunk
  const int rA = lane >> 2;       // fragment rows rA and rA + 8
  const int cq = (lane & 3) * 2;  // fragment column pair
  const int off = p.S - p.L;
  int lo_r[2], hi_r[2], row_i[2];
  bool live_r[2];
  int ks_u = 0, ke_u = p.S;  // EXT: the current unit's non-padding keys
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int r = rA + 8 * h;
    live_r[h] = r < p.R;
    const int i = live_r[h] ? (r % p.L) : 0;
    row_i[h] = i;
    lo_r[h] = (STREAM || p.mask_kind == MASK_WINDOW) ? i + off - p.window + 1 : 0;
    hi_r[h] = (p.mask_kind == MASK_NONE) ? p.S : min(p.S, i + off + 1);
  }

  uint32_t qa[E / 16][4];
  float o[EV / 8][4];
  float m_run[2], l_run[2];
  bool ok = true;

  auto load_q = [&](long long u) {
    const int n = static_cast<int>(u / p.H);
    const int kvh = static_cast<int>(u % p.H);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int r = rA + 8 * h;
      const __nv_bfloat16* qrow = nullptr;
      if (r < p.R) {
        const int hq = kvh * p.group + r / p.L;
        const int i = r % p.L;
        qrow = p.q + ((static_cast<size_t>(n) * p.Hq + hq) * p.L + i) * E;
      }
#pragma unroll
      for (int kk = 0; kk < E / 16; ++kk) {
        uint32_t lo = 0, hi = 0;
        if (qrow) {
          lo = *reinterpret_cast<const uint32_t*>(qrow + kk * 16 + cq);
          hi = *reinterpret_cast<const uint32_t*>(qrow + kk * 16 + 8 + cq);
        }
        qa[kk][h] = lo;       // a0 (row rA) / a1 (row rA+8)
        qa[kk][2 + h] = hi;   // a2 / a3
      }
    }
  };
  auto reset_state = [&]() {
#pragma unroll
    for (int t = 0; t < EV / 8; ++t) o[t][0] = o[t][1] = o[t][2] = o[t][3] = 0.f;
    m_run[0] = m_run[1] = -INFINITY;
    l_run[0] = l_run[1] = 0.f;
  };
  float* merge_o = reinterpret_cast<float*>(sp + C::OFF_MERGE);
  float* merge_ml = reinterpret_cast<float*>(sp + C::OFF_ML);
  // this warp's state -> its slot wq of the shared merge buffer (l summed over the quad)
  auto store_state = [&]() {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float l = l_run[h];
      l += __shfl_xor_sync(0xffffffffu, l, 1);
      l += __shfl_xor_sync(0xffffffffu, l, 2);
      const int r = rA + 8 * h;
      if ((lane & 3) == 0) {
        merge_ml[(wq * 16 + r) * 2 + 0] = m_run[h];
        merge_ml[(wq * 16 + r) * 2 + 1] = l;
      }
#pragma unroll
      for (int t = 0; t < EV / 8; ++t) {
        merge_o[(wq * 16 + r) * EV + t * 8 + cq] = o[t][2 * h];
        merge_o[(wq * 16 + r) * EV + t * 8 + cq + 1] = o[t][2 * h + 1];
      }
    }
  };
  auto flush = [&](long long u) {
    if constexpr (NGRP == 2) {
      // group 1 hands its state to group 0 through the buffer: warp wq of group 0 merges slot
      // wq (the same keys of the other chunks) into its registers
      if (grp == 1) store_state();
      consumer_bar<NCT>();
      if (grp == 0) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int r = rA + 8 * h;
          float l = l_run[h];
          l += __shfl_xor_sync(0xffffffffu, l, 1);
          l += __shfl_xor_sync(0xffffffffu, l, 2);
          const float m1 = merge_ml[(wq * 16 + r) * 2 + 0], l1 = merge_ml[(wq * 16 + r) * 2 + 1];
          const float M = fmaxf(m_run[h], m1);
          const float a0 = m_run[h] == -INFINITY ? 0.f : ex2(m_run[h] - M);
          const float a1 = m1 == -INFINITY ? 0.f : ex2(m1 - M);
#pragma unroll
          for (int t = 0; t < EV / 8; ++t) {
            o[t][2 * h] = fmaf(o[t][2 * h], a0, a1 * merge_o[(wq * 16 + r) * EV + t * 8 + cq]);
            o[t][2 * h + 1] = fmaf(o[t][2 * h + 1], a0, a1 * merge_o[(wq * 16 + r) * EV + t * 8 + cq + 1]);
          }
          m_run[h] = M;
          // the merged row sum, held by lane 0 of the quad so that the next quad sum restores it
          l_run[h] = (lane & 3) == 0 ? fmaf(l, a0, l1 * a1) : 0.f;
        }
      }
      consumer_bar<NCT>();
    }
    if (grp == 0) store_state();
    consumer_bar<NCT>();
    const size_t slot = static_cast<size_t>(blockIdx.x) + static_cast<size_t>(u);
    for (int x = threadIdx.x; x < p.R * EV; x += NCT) {
      const int r = x / EV, e = x % EV;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < DWARPS; ++w) M = fmaxf(M, merge_ml[(w * 16 + r) * 2]);
      float acc = 0.f, l = 0.f;
      if (M != -INFINITY) {
#pragma unroll
        for (int w = 0; w < DWARPS; ++w) {
          const float a = ex2(merge_ml[(w * 16 + r) * 2] - M);
          acc = fmaf(a, merge_o[(w * 16 + r) * EV + e], acc);
          l = fmaf(a, merge_ml[(w * 16 + r) * 2 + 1], l);
        }
      }
      p.ws_acc[(slot * 16 + r) * EV + e] = acc;
      if (e == 0) {
        p.ws_ml[(slot * 16 + r) * 2 + 0] = M;
        p.ws_ml[(slot * 16 + r) * 2 + 1] = l;
      }
    }
    // the CTA that finishes the unit's last segment merges all of its partials:
    // publish this partial, count it, and let the count's last arrival combine
    __threadfence();
    consumer_bar<NCT>();
    if (threadIdx.x == 0) {
      unsigned int* counters = reinterpret_cast<unsigned int*>(p.ws_ml + (static_cast<size_t>(p.G) + p.n_units) * 32);
      const long long nseg = cta_of(u * p.nc + p.nc - 1, p.T, p.G) - cta_of(u * p.nc, p.T, p.G) + 1;
      *last_flag = atomicAdd(counters + u, 1u) == static_cast<unsigned int>(nseg - 1) ? 1 : 0;
    }
    consumer_bar<NCT>();
    if (*last_flag) {
      __threadfence();
      for (int r = warp; r < p.R; r += NCW) combine_row<EV>(p, u, r, lane);
    }
    consumer_bar<NCT>();
  };

  // the units of this CTA's chunk range in order; every consumer warp walks all of them and
  // meets the others at each unit's flush
  for (long long cu = c_begin; cu < c_end;) {
    const long long u = cu / p.nc;
    const long long cu_end = min(c_end, (u + 1) * p.nc);
    load_q(u);
    reset_state();
    if constexpr (EXT) {
      const int n = static_cast<int>(u / p.H);
      ks_u = ga.kv_start ? __ldg(ga.kv_start + n) : 0;
      ke_u = ga.kv_end ? __ldg(ga.kv_end + n) : p.S;
    }
    const int first = (grp - static_cast<int>((cu - c_begin) % NGRP) + NGRP) % NGRP;
  for (long long c = cu + first; c < cu_end; c += NGRP) {
    const int idx = static_cast<int>(c - c_begin);
    const int s = idx % C::NSTAGE;
    const bool w_ok = mbar_wait(full_bar(s), (idx / C::NSTAGE) & 1);
    if (!__all_sync(0xffffffffu, w_ok)) {
      *abort_flag = 1;
      ok = false;
      break;
    }
    const uint32_t kbuf = sb + C::OFF_STAGES + s * C::STAGE_BYTES;
    const uint32_t vbuf = kbuf + C::K_BYTES;
    const int j0 = wq * 16;  // this warp's keys within the chunk
    const int key0 = GATHER ? 0 : chunk_key0<STREAM>(p, static_cast<int>(c % p.nc)) + j0;
    const int* keys_c = reinterpret_cast<const int*>(sp + C::OFF_KEYS) + s * DC + j0;  // GATHER

    // S = Q K^T for 16 keys (two n-tiles of 8).  Lane l holds dimensions
    // 2(l%4) + {0, 1, 8, 9} of each 16-wide slice for key l/4 of n-tile 0 (b0, b1)
    // and key 8 + l/4 of n-tile 1 (b2, b3).  RBF: in the order {b0, b2, b1, b3} the
    // same registers are the A fragment of the 16 keys x 16 dimensions block, so two
    // more MMAs accumulate the 16 x 16 Gram block K K^T, whose diagonal is ||k||^2
    float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    float gram[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};  // keys x keys 0-7, keys x keys 8-15
    {
      const int mat = lane >> 3;
      const int krow = j0 + (mat >> 1) * 8 + (lane & 7);
#pragma unroll
      for (int kk = 0; kk < E / 16; ++kk) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(kbuf + sw_off(krow, kk * 2 + (mat & 1)), b0, b1, b2, b3);
        mma16816(sc[0], qa[kk], b0, b1);
        mma16816(sc[1], qa[kk], b2, b3);
        if constexpr (RBF) {
          const uint32_t ka[4] = {b0, b2, b1, b3};
          mma16816(gram[0], ka, b0, b1);
          mma16816(gram[1], ka, b2, b3);
        }
      }
    }
    // RBF: each lane fetches the norms of the keys in its accumulator fragment (keys
    // t*8 + cq + {0, 1}).  Gram entry (i, i) of the first block sits in register i % 2 of
    // lane 9 (i / 2) + 4 (i % 2); entry (8 + i, 8 + i) of the second in register 2 + i % 2
    // of the same lane (the C fragment: lane 4g + u holds rows g, g + 8 and columns 2u, 2u + 1)
    float kn[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
    if constexpr (RBF) {
      const int src = 9 * (lane & 3);  // cq / 2 = lane % 4
      kn[0][0] = __shfl_sync(0xffffffffu, gram[0][0], src);
      kn[0][1] = __shfl_sync(0xffffffffu, gram[0][1], src + 4);
      kn[1][0] = __shfl_sync(0xffffffffu, gram[1][2], src);
      kn[1][1] = __shfl_sync(0xffffffffu, gram[1][3], src + 4);
    }
    // logits in base 2 (rbf: 2 scale q.k - scale ||k||^2), masks and bias
    const bool need_mask = GATHER || EXT || p.mask_kind != MASK_NONE || p.bias != nullptr || key0 + 16 > p.S;
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int h = e >> 1;
        float zz = RBF ? fmaf(sc[t][e], 2.f * p.c_dot, -kn[t][e & 1] * p.c_dot) : sc[t][e] * p.c_dot;
        if (need_mask) {
          const int key = GATHER ? keys_c[t * 8 + cq + (e & 1)] : key0 + t * 8 + cq + (e & 1);
          if constexpr (GATHER) {
            if (key < 0 || key < lo_r[h] || key >= hi_r[h]) zz = -INFINITY;  // -1: no key listed here
          } else if constexpr (STREAM) {
            if (key >= hi_r[h] || (key < lo_r[h] && key >= p.keep)) zz = -INFINITY;
          } else {
            if (key < lo_r[h] || key >= hi_r[h]) zz = -INFINITY;
          }
          if constexpr (EXT) {
            if (key < ks_u || key >= ke_u) zz = -INFINITY;
            if (ga.bits != nullptr && key < p.S &&
                !((__ldg(ga.bits + static_cast<size_t>(row_i[h]) * ga.words + (key >> 5)) >> (key & 31)) & 1u))
              zz = -INFINITY;
          }
          if (p.bias != nullptr && live_r[h] && key >= 0 && key < p.S)
            zz = fmaf(p.bias[static_cast<size_t>((rA + 8 * h) % p.L) * p.S + key], LOG2E, zz);
        }
        sc[t][e] = zz;
      }
    // online softmax (lazy rescale)
    float pr[2][4];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float mt = fmaxf(fmaxf(sc[0][2 * h], sc[0][2 * h + 1]), fmaxf(sc[1][2 * h], sc[1][2 * h + 1]));
      mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 1));
      mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 2));
      const float m_new = fmaxf(m_run[h], mt);
      if (m_new > m_run[h] + D_RESCALE_THRESHOLD) {
        const float alpha = ex2(m_run[h] - m_new);
        l_run[h] *= alpha;
#pragma unroll
        for (int t = 0; t < EV / 8; ++t) {
          o[t][2 * h] *= alpha;
          o[t][2 * h + 1] *= alpha;
        }
        m_run[h] = m_new;
      }
      const float mu = (m_run[h] == -INFINITY) ? 0.f : m_run[h];
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        pr[t][2 * h] = ex2(sc[t][2 * h] - mu);
        pr[t][2 * h + 1] = ex2(sc[t][2 * h + 1] - mu);
        l_run[h] += pr[t][2 * h] + pr[t][2 * h + 1];
      }
    }
    uint32_t pa[4];
    pa[0] = pack_bf16x2(pr[0][0], pr[0][1]);
    pa[1] = pack_bf16x2(pr[0][2], pr[0][3]);
    pa[2] = pack_bf16x2(pr[1][0], pr[1][1]);
    pa[3] = pack_bf16x2(pr[1][2], pr[1][3]);
    // O += P V
    {
      const int mat = lane >> 3;
      const int vrow = j0 + (mat & 1) * 8 + (lane & 7);
#pragma unroll
      for (int t = 0; t < EV / 8; t += 2) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(vbuf + sw_off(vrow, t + (mat >> 1)), b0, b1, b2, b3);
        mma16816(o[t], pa, b0, b1);
        mma16816(o[t + 1], pa, b2, b3);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty_bar(s));
  }
    // all consumer warps decide together: a failed wait in any of them ends the walk
    if (!consumer_bar_and<NCT>(ok)) break;
    flush(u);
    cu = cu_end;
  }
}

struct DecodePlan {
  int nc_head, kb_win, nc, G;
  long long T;
};

// Partial slots: one per (CTA, unit it touches), slot b + u.
size_t partial_slots(const DecodePlan& d, const AttnArgs& a) {
  return static_cast<size_t>(d.G) + static_cast<size_t>(a.N) * a.H;
}

// the even split of T chunks over a persistent grid, shared by both plans
void split(DecodePlan& d, const AttnArgs& a, int num_sms) {
  d.T = static_cast<long long>(a.N) * a.H * d.nc;
  d.G = static_cast<int>(d.T < num_sms ? d.T : num_sms);
}

// GATHER: a unit's chunks are 64 consecutive entries of its key list
DecodePlan plan_gather(const AttnArgs& a, int n_sel, int num_sms) {
  DecodePlan d{};
  d.nc = (n_sel + DC - 1) / DC;
  split(d, a, num_sms);
  return d;
}

DecodePlan plan(const AttnArgs& a, int num_sms) {
  DecodePlan d{};
  const int off = a.S - a.L;
  int lo = 0, hi = a.S;
  if (a.mask_kind != MASK_NONE) hi = a.S < off + a.L ? a.S : off + a.L;
  const int win_lo = off - a.window + 1 > 0 ? off - a.window + 1 : 0;
  if (a.mask_kind == MASK_WINDOW || (a.mask_kind == MASK_STREAM && a.keep == 0)) lo = win_lo;
  if (hi < 1) hi = 1;  // keep one chunk so every row gets a (fully masked) partial
  if (lo >= hi) lo = hi - 1;
  const int kb_hi = (hi + DC - 1) / DC;
  d.nc_head = 0;
  d.kb_win = lo / DC;
  if (a.mask_kind == MASK_STREAM && a.keep > 0) {
    // kept initial keys, then the window: the chunks between them are never read
    const int head = (a.keep + DC - 1) / DC;
    const int kb_w = win_lo / DC;
    if (kb_w > head && kb_w < kb_hi) {
      d.nc_head = head;
      d.kb_win = kb_w;
    }
  }
  d.nc = d.nc_head + (kb_hi - d.kb_win);
  split(d, a, num_sms);
  return d;
}

template <int E, int EV, bool STREAM, bool GATHER, bool EXT, bool RBF>
int launch_decode_impl(const AttnArgs& a, const ExtraArgs& ga, void* ws, size_t ws_bytes, int num_sms,
                       cudaStream_t stream) {
  using C = DCfg<E, EV, GATHER>;
  const DecodePlan d = GATHER ? plan_gather(a, ga.n_sel, num_sms) : plan(a, num_sms);
  const size_t slots = partial_slots(d, a);
  const size_t need = slots * 16 * (EV + 2) * sizeof(float) + static_cast<size_t>(a.N) * a.H * sizeof(unsigned int);
  if (ws_bytes < need) return -12;
  CUtensorMap tk{}, tv{};  // GATHER reads K and V through plain pointers; its maps stay unused
  if (!GATHER) {
    if (!make_map_rows(&tk, a.k, E, a.S, static_cast<long long>(a.N) * a.H, DC)) return -13;
    if (!make_map_rows(&tv, a.v, EV, a.S, static_cast<long long>(a.N) * a.H, DC)) return -13;
  }
  DecodeParams p{};
  p.q = static_cast<const __nv_bfloat16*>(a.q);
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.lse = a.lse;
  p.sink = a.sink;
  p.bias = a.bias;
  p.ws_acc = static_cast<float*>(ws);
  p.ws_ml = p.ws_acc + slots * 16 * EV;
  p.N = a.N;
  p.Hq = a.Hq;
  p.H = a.H;
  p.L = a.L;
  p.S = a.S;
  p.group = a.Hq / a.H;
  p.R = p.group * a.L;
  // the streaming mask without kept keys is the sliding window
  p.mask_kind = (a.mask_kind == MASK_STREAM && !STREAM) ? MASK_WINDOW : a.mask_kind;
  p.window = a.window;
  p.keep = STREAM ? a.keep : 0;
  p.nc_head = d.nc_head;
  p.kb_win = d.kb_win;
  p.nc = d.nc;
  p.T = d.T;
  p.G = d.G;
  p.n_units = a.N * a.H;
  p.c_dot = a.scale * LOG2E;
  auto kern = decode_partial_kernel<E, EV, STREAM, GATHER, EXT, RBF>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
    return -13;
  // per-unit arrival counters of the fused combine, after the partials
  unsigned int* counters = reinterpret_cast<unsigned int*>(p.ws_ml + slots * 32);
  if (cudaMemsetAsync(counters, 0, static_cast<size_t>(p.n_units) * sizeof(unsigned int), stream) != cudaSuccess)
    return -13;
  kern<<<d.G, GATHER ? (DWARPS + GWARPS) * 32 : DTHREADS, C::SMEM_BYTES, stream>>>(tk, tv, p, ga);
  return cudaGetLastError() == cudaSuccess ? 0 : -13;
}

}  // namespace

unsigned int take_status_decode(cudaStream_t s) { return take_device_status_local(s); }

bool decode_eligible(const AttnArgs& a) { return (a.Hq / a.H) * a.L <= 16; }

size_t decode_workspace_bytes(const AttnArgs& a, int num_sms) {
  const DecodePlan d = plan(a, num_sms);
  return partial_slots(d, a) * 16 * (a.Ev + 2) * sizeof(float) + static_cast<size_t>(a.N) * a.H * sizeof(unsigned int);
}

size_t decode_gather_workspace_bytes(const AttnArgs& a, int n_sel, int num_sms) {
  const DecodePlan d = plan_gather(a, n_sel, num_sms);
  return partial_slots(d, a) * 16 * (a.Ev + 2) * sizeof(float) + static_cast<size_t>(a.N) * a.H * sizeof(unsigned int);
}

int launch_decode_gather_bf16(const AttnArgs& a, const int* key_idx, int n_sel, void* ws, size_t ws_bytes,
                              int num_sms, cudaStream_t stream) {
  ExtraArgs ga{};
  ga.idx = key_idx;
  ga.k = static_cast<const __nv_bfloat16*>(a.k);
  ga.v = static_cast<const __nv_bfloat16*>(a.v);
  ga.n_sel = n_sel;
#define ATTN_GATHER_CASE(e, ev) \
  if (a.E == e && a.Ev == ev) return launch_decode_impl<e, ev, false, true, false, false>(a, ga, ws, ws_bytes, num_sms, stream);
  ATTN_GATHER_CASE(128, 128)
  ATTN_GATHER_CASE(64, 64)
  ATTN_GATHER_CASE(64, 128)
  ATTN_GATHER_CASE(128, 64)
#undef ATTN_GATHER_CASE
  return -4;
}

int launch_decode_bf16(const AttnArgs& a, void* ws, size_t ws_bytes, int num_sms, cudaStream_t stream) {
  // kept initial keys need the streaming mask test even where the plan makes no
  // head/window split (kept keys and window overlap: nc_head is then 0)
  const bool st = a.mask_kind == MASK_STREAM && a.keep > 0;
  const bool ext = a.mask_bits != nullptr || a.kv_start != nullptr || a.kv_end != nullptr;
  ExtraArgs xa{};
  xa.bits = a.mask_bits;
  xa.kv_start = a.kv_start;
  xa.kv_end = a.kv_end;
  xa.words = (a.S + 31) / 32;
#define ATTN_DECODE_CASE(e, ev)                                                                              \
  if (a.E == e && a.Ev == ev) {                                                                              \
    if (a.rbf) {                                                                                             \
      if (st) return launch_decode_impl<e, ev, true, false, false, true>(a, xa, ws, ws_bytes, num_sms, stream);  \
      if (ext) return launch_decode_impl<e, ev, false, false, true, true>(a, xa, ws, ws_bytes, num_sms, stream); \
      return launch_decode_impl<e, ev, false, false, false, true>(a, xa, ws, ws_bytes, num_sms, stream);         \
    }                                                                                                        \
    if (st) return launch_decode_impl<e, ev, true, false, false, false>(a, xa, ws, ws_bytes, num_sms, stream);   \
    if (ext) return launch_decode_impl<e, ev, false, false, true, false>(a, xa, ws, ws_bytes, num_sms, stream);  \
    return launch_decode_impl<e, ev, false, false, false, false>(a, xa, ws, ws_bytes, num_sms, stream);          \
  }
  ATTN_DECODE_CASE(128, 128)
  ATTN_DECODE_CASE(64, 64)
  ATTN_DECODE_CASE(64, 128)
  ATTN_DECODE_CASE(128, 64)
#undef ATTN_DECODE_CASE
  return -4;
}

}  // namespace attn

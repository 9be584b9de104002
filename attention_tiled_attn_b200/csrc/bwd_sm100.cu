// bf16 attention backward on tcgen05: dQ, dK, dV of the three score modes and
// the sink-logit gradient.
//
// The chain rule through the forward (page "Attention Sink" §4.2, §5: the sink
// and register tokens are learned, so training needs these gradients; page
// "Dot-Product Attention을 거리 기반 RBF-Attention으로 교체한 실험기": the RBF
// model is trained).  With the forward's lse (sink included), for one (batch,
// query head), query row i and key j:
//   P_ij  = 2^(z2_ij - lse2_i)            z2 = base-2 logit, lse2 = lse * log2e
//   D_i   = dout_i . out_i                (preprocess kernel)
//   dV_j += sum_i P_ij dout_i
//   dP_ij = dout_i . v_j
//   dS_ij = c_q P_ij (dP_ij - D_i)        c_q = scale (dot) or 2 scale (rbf)
//   dQ_i  = sum_j dS_ij k_j
//   dK_j += sum_i dS_ij q_i   (rbf: - k_j sum_i dS_ij)
//   dsink_h = -sum_i 2^(s2_h - lse2_i) D_i (preprocess kernel)
//
// One CTA per (batch, KV head, 128-key tile) walks the query tiles of every
// query head of its KV group that can see the tile, so dK and dV accumulate in
// tensor memory and are stored once; dQ is accumulated in global memory with
// vector reductions.  Per query tile five tcgen05 MMAs (M = N = 128):
//   S^T  = K Q^T        (SS)      into TMEM columns [0, 128)
//   dP^T = V dO^T       (SS)      into [128, 256)
//   dV  += P^T dO       (TS: P^T as bf16 in [0, 64), dO MN-major)
//   dK  += dS^T Q       (TS: dS^T as bf16 in [128, 192), Q MN-major)
//   dQ   = dS K         (SS: dS written to shared memory by the compute warps in
//                        the K-major layout the forward uses for Q; K MN-major)
//                        into [0, E)
// dV and dK live in [256, 256 + Ev) and [256 + Ev, 256 + Ev + E).  The dQ MMA
// reuses the S^T columns; tcgen05 MMAs of one thread run in issue order, so it
// follows the dV MMA that reads P^T there.
//
// Warps: 0-3 compute (thread = TMEM lane: a key row of S^T / dP^T, a query row
// of dQ), 4 TMA producer, 5 MMA issuer.  Every wait is bounded.

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kernels.h"
#include "ptx_sm100.cuh"

namespace attn {

namespace {

constexpr int TB = 128;  // keys per CTA tile and queries per query tile
constexpr int BTHREADS = 6 * 32;

// tcgen05 instruction descriptor with the A major bit as well (bit 15: MN-major A)
__host__ __device__ constexpr uint32_t idesc_ab(uint32_t M, uint32_t N, uint32_t a_mn, uint32_t b_mn) {
  return idesc_bf16_f32(M, N, b_mn) | (a_mn << 15);
}

template <int E, int EV>
struct BCfg {
  static constexpr int K_BYTES = TB * E * 2;
  static constexpr int V_BYTES = TB * EV * 2;
  static constexpr int Q_BYTES = TB * E * 2;
  static constexpr int DO_BYTES = TB * EV * 2;
  static constexpr int NSTAGE = 2;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + K_BYTES;
  static constexpr int OFF_Q = OFF_V + V_BYTES;                       // [NSTAGE] Q tiles
  static constexpr int OFF_DO = OFF_Q + NSTAGE * Q_BYTES;             // [NSTAGE] dO tiles
  static constexpr int OFF_DS = OFF_DO + NSTAGE * DO_BYTES;           // dS, 128 queries x 128 keys, K-major
  static constexpr int OFF_BAR = OFF_DS + TB * TB * 2;
  static constexpr int NBAR = 1 + 2 * NSTAGE + 6;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  // barriers
  static constexpr int B_KV = 0, B_QFULL = 1, B_QEMPTY = 1 + NSTAGE, B_SFULL = 1 + 2 * NSTAGE;
  static constexpr int B_PFULL = B_SFULL + 1, B_DQFULL = B_SFULL + 2, B_DQEMPTY = B_SFULL + 3;
  static constexpr int B_DKV = B_SFULL + 4, B_DRAIN = B_SFULL + 5;
  // TMEM columns
  static constexpr uint32_t T_S = 0, T_DP = 128, T_DV = 256, T_DK = 256 + EV;
  static constexpr uint32_t IDESC_S = idesc_ab(TB, TB, 0, 0);      // K Q^T and V dO^T
  static constexpr uint32_t IDESC_DV = idesc_ab(TB, EV, 0, 1);     // P^T dO
  static constexpr uint32_t IDESC_DK = idesc_ab(TB, E, 0, 1);      // dS^T Q
  static constexpr uint32_t IDESC_DQ = idesc_ab(TB, E, 0, 1);      // dS K
};

struct BwdParams {
  const float* lse2;   // [N*Hq*Lp] the forward's lse * log2e, -inf past L (Lp = L rounded up to 128)
  const float* dsum;   // [N*Hq*Lp] D = dout . out, 0 past L
  float* dq;           // [N*Hq*L*E], accumulated (zeroed by the launcher)
  float* dk;           // [N*H*S*E]
  float* dv;           // [N*H*S*Ev]
  int N, Hq, H, L, S, group, Lp;
  int mask_kind, window;
  int keep;             // MASK_STREAM: kept initial keys
  const uint32_t* bits;  // [L][words] keep bits, or nullptr
  const int* kv_start;   // [N] or nullptr
  const int* kv_end;     // [N] or nullptr
  int words;
  int rbf;
  float c_z;           // base-2 logit per unit of q.k: scale*log2e (dot) or 2*scale*log2e (rbf)
  float c_kn;          // rbf: scale*log2e per unit of |k|^2
  float c_q;           // dS scale: scale (dot) or 2*scale (rbf)
};

__device__ __forceinline__ bool bwait(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
  if (*abort_flag) return false;
  if (mbar_wait(bar, parity)) return true;
  *abort_flag = 1;
  return false;
}

__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// query tiles of head-local rows that can see some key of [k0, k0 + TB)
template <bool MX>
__device__ __forceinline__ void query_tiles(const BwdParams& p, int k0, int& qt_lo, int& qt_hi) {
  const int off = p.S - p.L;
  int lo = 0, hi = p.L;  // query rows [lo, hi)
  if (p.mask_kind != MASK_NONE) lo = max(0, k0 - off);  // i' >= j
  // i' - j < W, except that kept keys (streaming) stay visible to every later query
  if (p.mask_kind == MASK_WINDOW || (MX && p.mask_kind == MASK_STREAM && k0 >= p.keep))
    hi = min(p.L, k0 + TB - 1 + p.window - off);
  qt_lo = lo / TB;
  qt_hi = hi > lo ? (hi + TB - 1) / TB : qt_lo;
}

// MX: the streaming mask, keep bits or key padding is in use (a separate instantiation,
// so the plain masks keep their own register allocation)
template <int E, int EV, bool MX>
__global__ void __launch_bounds__(BTHREADS, 1)
    bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
               const BwdParams p) {
  using C = BCfg<E, EV>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t sb = smem_u32(smem_raw);
  if (sb & 1023u) {  // the layout needs a 1024-byte aligned base; report instead of overrunning
    if (threadIdx.x == 0) record_timeout();
    return;
  }
  uint8_t* sp = smem_raw;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sp + C::OFF_MISC);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sp + C::OFF_MISC + 4);
  auto bar = [&](int i) -> uint32_t { return sb + C::OFF_BAR + 8u * i; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // key-tile-major numbering: under a causal mask the early key tiles see the most
  // query tiles, so the heaviest CTAs are launched first
  const int nh_total = p.N * p.H;
  const int kt = blockIdx.x / nh_total;
  const int nh = blockIdx.x % nh_total;  // n * H + kvh
  const int n = nh / p.H, kvh = nh % p.H;
  const int k0 = kt * TB;
  int qt_lo, qt_hi;
  query_tiles<MX>(p, k0, qt_lo, qt_hi);
  // key padding of this batch: a key tile wholly outside [ks, ke) has zero gradients
  int ks = 0, ke = p.S;
  if constexpr (MX) {
    if (p.kv_start) ks = max(0, p.kv_start[n]);
    if (p.kv_end) ke = min(p.S, p.kv_end[n]);
    if (k0 + TB <= ks || k0 >= ke) qt_hi = qt_lo;
  }
  const int n_qt = qt_hi - qt_lo;
  const int n_it = n_qt * p.group;  // (query head of the group, query tile) pairs

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(bar(C::B_KV), 1);
    for (int s = 0; s < C::NSTAGE; ++s) {
      mbar_init(bar(C::B_QFULL + s), 1);
      mbar_init(bar(C::B_QEMPTY + s), 1);
    }
    mbar_init(bar(C::B_SFULL), 1);
    mbar_init(bar(C::B_PFULL), 128);
    mbar_init(bar(C::B_DQFULL), 1);
    mbar_init(bar(C::B_DQEMPTY), 128);
    mbar_init(bar(C::B_DKV), 1);
    mbar_init(bar(C::B_DRAIN), 1);
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ================= TMA producer =================
    if (lane == 0) {
      mbar_arrive_expect_tx(bar(C::B_KV), C::K_BYTES + C::V_BYTES);
      for (int b = 0; b < E / 64; ++b) tma_load_3d(sb + C::OFF_K + b * (TB * 128), &tm_k, bar(C::B_KV), b * 64, k0, nh);
      for (int b = 0; b < EV / 64; ++b)
        tma_load_3d(sb + C::OFF_V + b * (TB * 128), &tm_v, bar(C::B_KV), b * 64, k0, nh);
      int issued = 0;
      for (int it = 0; it < n_it; ++it) {
        const int s = it % C::NSTAGE;
        if (!bwait(bar(C::B_QEMPTY + s), ((it / C::NSTAGE) & 1) ^ 1, abort_flag)) break;
        const int hq = kvh * p.group + it / n_qt;
        const int q0 = (qt_lo + it % n_qt) * TB;
        const int qrow = n * p.Hq + hq;
        mbar_arrive_expect_tx(bar(C::B_QFULL + s), C::Q_BYTES + C::DO_BYTES);
        for (int b = 0; b < E / 64; ++b)
          tma_load_3d(sb + C::OFF_Q + s * C::Q_BYTES + b * (TB * 128), &tm_q, bar(C::B_QFULL + s), b * 64, q0, qrow);
        for (int b = 0; b < EV / 64; ++b)
          tma_load_3d(sb + C::OFF_DO + s * C::DO_BYTES + b * (TB * 128), &tm_do, bar(C::B_QFULL + s), b * 64, q0,
                      qrow);
        issued = it + 1;
      }
      // drain: every issued copy has landed before exit
      mbar_wait(bar(C::B_KV), 0);
      for (int it = (issued > C::NSTAGE ? issued - C::NSTAGE : 0); it < issued; ++it)
        mbar_wait(bar(C::B_QFULL + it % C::NSTAGE), (it / C::NSTAGE) & 1);
    }
  } else if (warp == 5) {
    // ================= tcgen05 issuer =================
    if (lane == 0) {
      bool ok = bwait(bar(C::B_KV), 0, abort_flag);
      tc_fence_after();
      constexpr uint32_t hi = desc_hi_sw128(1024);
      const uint32_t k_lo_kmaj = desc_lo(sb + C::OFF_K, 16);
      const uint32_t v_lo_kmaj = desc_lo(sb + C::OFF_V, 16);
      const uint32_t k_lo_mn = desc_lo(sb + C::OFF_K, TB * 128);
      const uint32_t ds_lo_kmaj = desc_lo(sb + C::OFF_DS, 16);
      for (int it = 0; ok && it < n_it; ++it) {
        const int s = it % C::NSTAGE;
        if (!bwait(bar(C::B_QFULL + s), (it / C::NSTAGE) & 1, abort_flag)) break;
        if (it > 0 && !bwait(bar(C::B_DQEMPTY), (it - 1) & 1, abort_flag)) break;  // dQ of it-1 read
        tc_fence_after();
        const uint32_t q_lo_kmaj = desc_lo(sb + C::OFF_Q + s * C::Q_BYTES, 16);
        const uint32_t do_lo_kmaj = desc_lo(sb + C::OFF_DO + s * C::DO_BYTES, 16);
        // S^T = K Q^T, dP^T = V dO^T (K-major operands; K steps of 16 inside 64-column boxes)
#pragma unroll
        for (int kk = 0; kk < E / 16; ++kk) {
          const uint32_t koff = ((kk / 4) * (TB * 128) + (kk % 4) * 32) >> 4;
          mma_ss_h(tmem + C::T_S, k_lo_kmaj + koff, hi, q_lo_kmaj + koff, hi, C::IDESC_S, kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < EV / 16; ++kk) {
          const uint32_t koff = ((kk / 4) * (TB * 128) + (kk % 4) * 32) >> 4;
          mma_ss_h(tmem + C::T_DP, v_lo_kmaj + koff, hi, do_lo_kmaj + koff, hi, C::IDESC_S, kk > 0 ? 1u : 0u);
        }
        mma_commit(bar(C::B_SFULL));
        if (!bwait(bar(C::B_PFULL), it & 1, abort_flag)) break;
        tc_fence_after();
        // dV += P^T dO, dK += dS^T Q (A from TMEM: 8 columns per 16 queries; B MN-major: 16 rows per step)
        const uint32_t do_lo_mn = desc_lo(sb + C::OFF_DO + s * C::DO_BYTES, TB * 128);
        const uint32_t q_lo_mn = desc_lo(sb + C::OFF_Q + s * C::Q_BYTES, TB * 128);
#pragma unroll
        for (int kk = 0; kk < TB / 16; ++kk)
          mma_ts_h(tmem + C::T_DV, tmem + C::T_S + kk * 8, do_lo_mn + kk * 128, hi, C::IDESC_DV,
                   (it > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < TB / 16; ++kk)
          mma_ts_h(tmem + C::T_DK, tmem + C::T_DP + kk * 8, q_lo_mn + kk * 128, hi, C::IDESC_DK,
                   (it > 0 || kk > 0) ? 1u : 0u);
        // dQ = dS K: A = dS in shared memory (K-major over keys), B = K read MN-major (16 keys per step)
#pragma unroll
        for (int kk = 0; kk < TB / 16; ++kk) {
          const uint32_t koff = ((kk / 4) * (TB * 128) + (kk % 4) * 32) >> 4;
          mma_ss_h(tmem + C::T_S, ds_lo_kmaj + koff, hi, k_lo_mn + kk * 128, hi, C::IDESC_DQ, kk > 0 ? 1u : 0u);
        }
        mma_commit(bar(C::B_DQFULL));
        mma_commit(bar(C::B_QEMPTY + s));  // Q and dO of this stage are no longer read
      }
      mma_commit(bar(C::B_DKV));
      mma_commit(bar(C::B_DRAIN));
      mbar_wait(bar(C::B_DRAIN), 0);
    }
  } else {
    // ================= compute warps 0-3 =================
    const int t = threadIdx.x;  // TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const int j = k0 + t;       // this thread's key row of S^T / dP^T
    const int off = p.S - p.L;
    // rbf: the key-norm term of this key, in base-2 logit units
    float kn2 = 0.f;
    if (p.rbf) {
      const uint8_t* kt_s = sp + C::OFF_K;
      float acc = 0.f;
      const bool kv_ok = __all_sync(0xffffffffu, bwait(bar(C::B_KV), 0, abort_flag));
      if (kv_ok) {
#pragma unroll
        for (int bb = 0; bb < E / 64; ++bb)
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint4 w = *reinterpret_cast<const uint4*>(kt_s + bb * (TB * 128) + t * 128 + ((c ^ (t & 7)) << 4));
            const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float lo = __uint_as_float(ws[e] << 16), hi = __uint_as_float(ws[e] & 0xFFFF0000u);
              acc = fmaf(lo, lo, fmaf(hi, hi, acc));
            }
          }
      }
      kn2 = acc * p.c_kn;
    }
    float ds_rowsum = 0.f;  // rbf: sum_i dS_ij of this key
    bool ok = true;
    for (int it = 0; it < n_it; ++it) {
      const int hq = kvh * p.group + it / n_qt;
      const int q0 = (qt_lo + it % n_qt) * TB;
      const size_t rowbase = (static_cast<size_t>(n) * p.Hq + hq) * p.L;
      const size_t padbase = (static_cast<size_t>(n) * p.Hq + hq) * p.Lp + q0;  // 16-byte aligned
      if (!__all_sync(0xffffffffu, bwait(bar(C::B_SFULL), it & 1, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const bool key_ok = j < p.S;
      // dS element (query c, this key t) of the K-major tile: box t/64, row c, 16-byte unit (t%64)/8 swizzled by c
      uint8_t* ds_col = sp + C::OFF_DS + (t >> 6) * (TB * 128) + (t & 7) * 2;
      const int ds_unit = (t & 63) >> 3;
#pragma unroll 1
      for (int ch = 0; ch < TB / 32; ++ch) {
        // the chunk's lse2 and D (every thread reads the same 256 bytes: L1 broadcast), issued first
        float4 l4[8], d4[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          l4[u] = __ldg(reinterpret_cast<const float4*>(p.lse2 + padbase + ch * 32) + u);
          d4[u] = __ldg(reinterpret_cast<const float4*>(p.dsum + padbase + ch * 32) + u);
        }
        uint32_t sr[32], dr[32];
        tmem_ld32(tmem + lane_base + C::T_S + ch * 32, sr);
        tmem_ld32(tmem + lane_base + C::T_DP + ch * 32, dr);
        tmem_wait_ld();
        uint32_t pk[16], dk[16];
        float dsv[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int c = ch * 32 + e;
          const int i = q0 + c;
          const float4 lv = l4[e >> 2], dv4 = d4[e >> 2];
          const float l2 = (e & 3) == 0 ? lv.x : (e & 3) == 1 ? lv.y : (e & 3) == 2 ? lv.z : lv.w;
          const float dd = (e & 3) == 0 ? dv4.x : (e & 3) == 1 ? dv4.y : (e & 3) == 2 ? dv4.z : dv4.w;
          bool vis = key_ok && l2 != -INFINITY;  // -inf past L and on rows that see no key
          if (p.mask_kind != MASK_NONE) vis = vis && j <= i + off;
          if (p.mask_kind == MASK_WINDOW) vis = vis && (i + off - j) < p.window;
          if constexpr (MX) {
            if (p.mask_kind == MASK_STREAM) vis = vis && (j < p.keep || (i + off - j) < p.window);
            vis = vis && j >= ks && j < ke;
            // keep bit (i, j): the 32 lanes of a warp hold 32 consecutive keys, one word (broadcast)
            if (vis && p.bits != nullptr)
              vis = (__ldg(p.bits + static_cast<size_t>(i) * p.words + (j >> 5)) >> (j & 31)) & 1u;
          }
          const float z2 = fmaf(__uint_as_float(sr[e]), p.c_z, -kn2);
          const float pr = vis ? ex2(z2 - l2) : 0.f;
          const float ds = p.c_q * pr * (__uint_as_float(dr[e]) - dd);
          dsv[e] = ds;
          ds_rowsum += ds;
          sr[e] = __float_as_uint(pr);
        }
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          pk[e] = pack_bf16x2(__uint_as_float(sr[2 * e]), __uint_as_float(sr[2 * e + 1]));
          dk[e] = pack_bf16x2(dsv[2 * e], dsv[2 * e + 1]);
        }
        // P^T and dS^T as bf16 pairs: chunk ch goes to columns already read
        tmem_st16(tmem + lane_base + C::T_S + ch * 16, pk);
        tmem_st16(tmem + lane_base + C::T_DP + ch * 16, dk);
        // dS into the K-major shared tile: one bf16 per query row (a warp's 32 keys fill 64 contiguous bytes)
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int c = ch * 32 + e;
          *reinterpret_cast<__nv_bfloat16*>(ds_col + c * 128 + ((ds_unit ^ (c & 7)) << 4)) = __float2bfloat16_rn(dsv[e]);
        }
      }
      tmem_wait_st();
      fence_proxy_async_smem();  // the dS^T tile is read by the tensor core (async proxy)
      tc_fence_before();
      mbar_arrive(bar(C::B_PFULL));
      // dQ rows of this query tile: lane t = query q0 + t
      if (!__all_sync(0xffffffffu, bwait(bar(C::B_DQFULL), it & 1, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      {
        const int i = q0 + t;
        float* dq_row = p.dq + (rowbase + i) * E;
#pragma unroll 1
        for (int c = 0; c < E; c += 32) {
          uint32_t r[32];
          tmem_ld32(tmem + lane_base + C::T_S + c, r);
          tmem_wait_ld();
          if (i < p.L) {
#pragma unroll
            for (int e = 0; e < 32; e += 4)
              red_add_v4(dq_row + c + e, __uint_as_float(r[e]), __uint_as_float(r[e + 1]), __uint_as_float(r[e + 2]),
                         __uint_as_float(r[e + 3]));
          }
        }
      }
      tc_fence_before();
      mbar_arrive(bar(C::B_DQEMPTY));
    }
    // dK and dV of this key row
    ok = __all_sync(0xffffffffu, ok);
    if (ok && n_it > 0 && __all_sync(0xffffffffu, bwait(bar(C::B_DKV), 0, abort_flag))) {
      tc_fence_after();
      // tcgen05.ld is warp-collective: every lane loads, only rows j < S are stored
      const bool row_ok = j < p.S;
      float* dv_row = p.dv + (static_cast<size_t>(nh) * p.S + j) * EV;
      float* dk_row = p.dk + (static_cast<size_t>(nh) * p.S + j) * E;
#pragma unroll 1
      for (int c = 0; c < EV; c += 32) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_base + C::T_DV + c, r);
        tmem_wait_ld();
        if (row_ok) {
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(dv_row + c + e) = make_float4(
                __uint_as_float(r[e]), __uint_as_float(r[e + 1]), __uint_as_float(r[e + 2]), __uint_as_float(r[e + 3]));
        }
      }
      const uint8_t* kt_s = sp + C::OFF_K;
#pragma unroll 1
      for (int c = 0; c < E; c += 32) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_base + C::T_DK + c, r);
        tmem_wait_ld();
        float g[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) g[e] = __uint_as_float(r[e]);
        if (p.rbf) {
          // - k_j * sum_i dS_ij (k from the swizzled K tile: column c + e is 16-byte unit ((c+e)%64)/8 of box (c+e)/64)
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int col = c + 8 * u;
            const uint4 w = *reinterpret_cast<const uint4*>(kt_s + (col / 64) * (TB * 128) + t * 128 +
                                                            ((((col % 64) / 8) ^ (t & 7)) << 4));
            const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              g[8 * u + 2 * e] -= __uint_as_float(ws[e] << 16) * ds_rowsum;
              g[8 * u + 2 * e + 1] -= __uint_as_float(ws[e] & 0xFFFF0000u) * ds_rowsum;
            }
          }
        }
        if (row_ok) {
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(dk_row + c + e) = make_float4(g[e], g[e + 1], g[e + 2], g[e + 3]);
        }
      }
    } else if (n_it == 0 && j < p.S) {
      // no query sees this key tile: its gradients are zero
      float* dv_row = p.dv + (static_cast<size_t>(nh) * p.S + j) * EV;
      float* dk_row = p.dk + (static_cast<size_t>(nh) * p.S + j) * E;
      for (int c = 0; c < EV; ++c) dv_row[c] = 0.f;
      for (int c = 0; c < E; ++c) dk_row[c] = 0.f;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// D_i = dout_i . out_i (fp32), lse2_i = lse_i * log2e, both padded per head to Lp
// rows (D = 0, lse2 = -inf past L), and the sink gradient -sum_i 2^(s2 - lse2_i) D_i.
// One warp per padded row.
template <int EV>
__global__ void __launch_bounds__(256) bwd_pre_kernel(const __nv_bfloat16* __restrict__ out,
                                                      const __nv_bfloat16* __restrict__ dout,
                                                      const float* __restrict__ lse, const float* __restrict__ sink,
                                                      float* __restrict__ dsum, float* __restrict__ lse2,
                                                      float* __restrict__ dsink, int Hq, int L, int Lp,
                                                      long long prows) {
  const long long pr = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (pr >= prows) return;
  const long long head = pr / Lp;
  const int i = static_cast<int>(pr % Lp);
  if (i >= L) {
    if (lane == 0) {
      dsum[pr] = 0.f;
      lse2[pr] = -INFINITY;
    }
    return;
  }
  const long long r = head * L + i;
  float acc = 0.f;
  for (int e = lane * 2; e < EV; e += 64) {
    const __nv_bfloat162 o2 = *reinterpret_cast<const __nv_bfloat162*>(out + r * EV + e);
    const __nv_bfloat162 d2 = *reinterpret_cast<const __nv_bfloat162*>(dout + r * EV + e);
    acc = fmaf(__low2float(o2), __low2float(d2), acc);
    acc = fmaf(__high2float(o2), __high2float(d2), acc);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) {
    const float l = lse[r];
    dsum[pr] = acc;
    lse2[pr] = l * LOG2E;
    if (sink != nullptr && dsink != nullptr) {  // a caller may pass sink logits without asking for dsink
      const int hq = static_cast<int>(head % Hq);
      if (l != -INFINITY) atomicAdd(dsink + hq, -ex2((sink[hq] - l) * LOG2E) * acc);
    }
  }
}

template <int E, int EV>
int launch_bwd_impl(const BwdArgs& a, float* ws, cudaStream_t stream) {
  using C = BCfg<E, EV>;
  const long long rows = static_cast<long long>(a.N) * a.Hq * a.L;
  const int Lp = (a.L + TB - 1) / TB * TB;
  const long long prows = static_cast<long long>(a.N) * a.Hq * Lp;
  float* dsum = ws;
  float* lse2 = ws + prows;
  if (cudaMemsetAsync(a.dq, 0, static_cast<size_t>(rows) * E * sizeof(float), stream) != cudaSuccess) return -13;
  if (a.dsink && cudaMemsetAsync(a.dsink, 0, static_cast<size_t>(a.Hq) * sizeof(float), stream) != cudaSuccess)
    return -13;
  bwd_pre_kernel<EV><<<static_cast<unsigned>((prows + 7) / 8), 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(a.out), static_cast<const __nv_bfloat16*>(a.dout), a.lse, a.sink, dsum, lse2,
      a.dsink, a.Hq, a.L, Lp, prows);
  if (cudaGetLastError() != cudaSuccess) return -13;
  CUtensorMap tq, tk, tv, tdo;
  if (!make_map_rows(&tq, a.q, E, a.L, static_cast<long long>(a.N) * a.Hq, TB)) return -13;
  if (!make_map_rows(&tdo, a.dout, EV, a.L, static_cast<long long>(a.N) * a.Hq, TB)) return -13;
  if (!make_map_rows(&tk, a.k, E, a.S, static_cast<long long>(a.N) * a.H, TB)) return -13;
  if (!make_map_rows(&tv, a.v, EV, a.S, static_cast<long long>(a.N) * a.H, TB)) return -13;
  BwdParams p{};
  p.lse2 = lse2;
  p.dsum = dsum;
  p.Lp = Lp;
  p.dq = a.dq;
  p.dk = a.dk;
  p.dv = a.dv;
  p.N = a.N;
  p.Hq = a.Hq;
  p.H = a.H;
  p.L = a.L;
  p.S = a.S;
  p.group = a.Hq / a.H;
  p.mask_kind = a.mask_kind;
  p.window = a.window;
  p.keep = a.keep;
  p.bits = a.mask_bits;
  p.kv_start = a.kv_start;
  p.kv_end = a.kv_end;
  p.words = (a.S + 31) / 32;
  p.rbf = a.rbf ? 1 : 0;
  p.c_z = (a.rbf ? 2.f : 1.f) * a.scale * LOG2E;
  p.c_kn = a.scale * LOG2E;
  p.c_q = (a.rbf ? 2.f : 1.f) * a.scale;
  const bool mx = a.mask_kind == MASK_STREAM || a.mask_bits || a.kv_start || a.kv_end;
  auto kern = mx ? bwd_kernel<E, EV, true> : bwd_kernel<E, EV, false>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess)
    return -13;
  const long long grid = static_cast<long long>(a.N) * a.H * ((a.S + TB - 1) / TB);
  if (grid > 0x7fffffffLL) return -2;
  kern<<<static_cast<unsigned>(grid), BTHREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, tdo, p);
  return cudaGetLastError() == cudaSuccess ? 0 : -13;
}

}  // namespace

unsigned int take_status_bwd(cudaStream_t s) { return take_device_status_local(s); }

size_t bwd_workspace_bytes(const BwdArgs& a) {
  const size_t Lp = (static_cast<size_t>(a.L) + TB - 1) / TB * TB;
  return 2 * static_cast<size_t>(a.N) * a.Hq * Lp * sizeof(float);  // D and lse2, padded per head
}

int launch_bwd_bf16(const BwdArgs& a, void* workspace, cudaStream_t stream) {
  float* dsum = static_cast<float*>(workspace);
  if (a.E == 128 && a.Ev == 128) return launch_bwd_impl<128, 128>(a, dsum, stream);
  if (a.E == 64 && a.Ev == 64) return launch_bwd_impl<64, 64>(a, dsum, stream);
  if (a.E == 64 && a.Ev == 128) return launch_bwd_impl<64, 128>(a, dsum, stream);
  if (a.E == 128 && a.Ev == 64) return launch_bwd_impl<128, 64>(a, dsum, stream);
  return -4;
}

}  // namespace attn

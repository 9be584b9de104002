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
// One CTA per (batch, KV head, 128-key tile) walks the 64-query tiles of every
// query head of its KV group that can see the key tile, so dK and dV accumulate
// in tensor memory and are stored once; dQ is accumulated in global memory with
// bulk tensor reduce-adds.  Per query tile b = it % 2 (two tiles in flight) five tcgen05 MMAs,
// M = 128 keys (or head dimensions for dQ^T):
//   S^T  = K Q^T      (SS, N = 64)             into TMEM columns S_b = [64 b, 64 b + 64)
//   dP^T = V dO^T     (SS, N = 64)             into DP_b = [128 + 64 b, 192 + 64 b)
//   dQ^T = K^T dS'^T  (SS, N = 64: K read MN-major, dS'^T MN-major)  into DP_b once dP^T is read
//   dV  += P^T dO     (TS: P^T as bf16 pairs over the S_b columns, dO MN-major)
//   dK  += dS'^T Q    (SS: dS'^T K-major, Q MN-major)
// with dS' = dS / c_q; the factor c_q is applied where dQ and dK leave the kernel.
// dS'^T (128 keys x 64 queries, bf16) is written to shared memory once per tile
// (two buffers): read K-major it is the A operand of dK, read MN-major the B
// operand of dQ^T.  dQ^T puts a head-dimension index on each TMEM lane; the readout
// warpgroup stages it in shared memory as fp32 [query][E] and adds each 32-query half
// into dq with one bulk tensor reduce-add (the tensor map drops rows past L).  dV
// and dK live in [256, 256 + Ev) and [256 + Ev, 256 + Ev + E).  tcgen05 MMAs of
// one thread run in issue order, so S^T of tile it + 2 may be issued into the
// columns the dV MMA of tile it still reads.
//
// Warps: 0-7 compute in two warpgroups (thread = TMEM lane = key row; warpgroup g
// takes queries [32 g, 32 g + 32) of each tile), 8-11 read dQ^T out (thread =
// head-dimension index; their elected thread also issues the dP^T that reuses the
// columns just read), 12 TMA producer (Q, dO and the tile's lse2 and D), 13 the MMA
// issuer of dQ^T, 14 the MMA issuer of S^T, dV and dK.  Every wait is bounded.

#include <climits>
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kernels.h"
#include "ptx_sm100.cuh"

namespace attn {

namespace {

constexpr int TB = 128;           // keys per CTA tile
constexpr int QT = 64;            // queries per query tile
constexpr int N_COMPUTE = 256;    // two warpgroups
constexpr int W_DQ = N_COMPUTE / 32;  // first dQ readout warp
constexpr int W_PRODUCER = W_DQ + 4;
constexpr int W_ISSUER = W_PRODUCER + 1;   // dP^T and dQ^T: the MMAs a warpgroup waits for
constexpr int W_ISSUER2 = W_ISSUER + 1;    // S^T, dV and dK: the MMAs with slack
constexpr int BTHREADS = (W_ISSUER2 + 1) * 32;

// tcgen05 instruction descriptor with the A major bit as well (bit 15: MN-major A)
__host__ __device__ constexpr uint32_t idesc_ab(uint32_t M, uint32_t N, uint32_t a_mn, uint32_t b_mn) {
  return idesc_bf16_f32(M, N, b_mn) | (a_mn << 15);
}

template <int E, int EV>
struct BCfg {
  static constexpr int K_BYTES = TB * E * 2;
  static constexpr int V_BYTES = TB * EV * 2;
  static constexpr int Q_BYTES = QT * E * 2;
  static constexpr int DO_BYTES = QT * EV * 2;
  static constexpr int LD_BYTES = 2 * QT * 4;                          // lse2 and D of the tile
  static constexpr int NSTAGE = 3;
  static constexpr int DS_BYTES = TB * QT * 2;                         // one dS'^T buffer
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + K_BYTES;
  static constexpr int OFF_Q = OFF_V + V_BYTES;                        // [NSTAGE] Q tiles
  static constexpr int OFF_DO = OFF_Q + NSTAGE * Q_BYTES;              // [NSTAGE] dO tiles
  static constexpr int OFF_DS = OFF_DO + NSTAGE * DO_BYTES;            // [2] dS'^T
  static constexpr int OFF_DQS = OFF_DS + 2 * DS_BYTES;                // dQ staging, [64 queries][E] fp32
  static constexpr int DQS_BYTES = QT * E * 4;
  static constexpr int OFF_LD = OFF_DQS + DQS_BYTES;                   // [NSTAGE] lse2[64], D[64]
  static constexpr int OFF_BAR = OFF_LD + NSTAGE * LD_BYTES;
  // barriers
  static constexpr int B_KV = 0, B_QFULL = 1, B_QEMPTY = 1 + NSTAGE, B_SFULL = 1 + 2 * NSTAGE;
  static constexpr int B_PFULL = B_SFULL + 2, B_DQFULL = B_SFULL + 4;
  static constexpr int B_DKV = B_SFULL + 6, B_DRAIN = B_SFULL + 7;  // B_DRAIN: [3], one per issuing thread
  static constexpr int NBAR = B_DRAIN + 3;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(E >= 64 && E <= TB, "dQ^T takes the head dimension as M = 128");
  static_assert(DS_BYTES >= 2 * TB * 4, "the rbf row-sum exchange reuses a dS'^T buffer");
  // TMEM columns
  static constexpr uint32_t T_S = 0, T_DP = 128, T_DV = 256, T_DK = 256 + EV;
  static constexpr uint32_t IDESC_S = idesc_ab(TB, QT, 0, 0);      // K Q^T and V dO^T
  static constexpr uint32_t IDESC_DV = idesc_ab(TB, EV, 0, 1);     // P^T dO
  static constexpr uint32_t IDESC_DK = idesc_ab(TB, E, 0, 1);      // dS'^T Q
  static constexpr uint32_t IDESC_DQ = idesc_ab(TB, QT, 1, 1);     // K^T dS'^T (rows >= E unused when E = 64)
};

struct BwdParams {
  const float* lse2;   // [N*Hq*Lp] the forward's lse * log2e; +inf past L and on rows that see no key
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

// the two compute warpgroups only (named barrier 1); the dQ readout warpgroup only (named barrier 2)
__device__ __forceinline__ void compute_bar() { asm volatile("bar.sync 1, %0;" ::"n"(N_COMPUTE) : "memory"); }
__device__ __forceinline__ void dq_bar() { asm volatile("bar.sync 2, 128;" ::: "memory"); }
// the same barrier returning the AND of every thread's flag (a uniform decision)
__device__ __forceinline__ bool dq_bar_and(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.and.pred p, 2, 128, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v))
      : "memory");
  return r != 0;
}

// Bulk tensor reduce-add (fp32, tile mode, no multicast) of a shared-memory box into global
// memory at coordinates (c0, c1, c2); elements outside the tensor are skipped.
__device__ __forceinline__ void bulk_reduce_add_3d(const CUtensorMap* map, uint32_t src, int c0, int c1, int c2) {
  asm volatile("cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(src), "r"(c0), "r"(c1), "r"(c2)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// every committed bulk operation of this thread has finished reading shared memory
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// every committed bulk operation of this thread has completed
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Plain (non-multicast) bulk copy of `bytes` (a multiple of 16, both addresses
// 16-byte aligned) from global to this CTA's shared memory, completing on `bar`.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

// query tiles (of QT rows, head-local) that can see some key of [k0, k0 + TB)
template <bool MX>
__device__ __forceinline__ void query_tiles(const BwdParams& p, int k0, int& qt_lo, int& qt_hi) {
  const int off = p.S - p.L;
  int lo = 0, hi = p.L;  // query rows [lo, hi)
  if (p.mask_kind != MASK_NONE) lo = max(0, k0 - off);  // i' >= j
  // i' - j < W, except that kept keys (streaming) stay visible to every later query
  if (p.mask_kind == MASK_WINDOW || (MX && p.mask_kind == MASK_STREAM && k0 >= p.keep))
    hi = min(p.L, k0 + TB - 1 + p.window - off);
  qt_lo = lo / QT;
  qt_hi = hi > lo ? (hi + QT - 1) / QT : qt_lo;
}

// One warp's 32 x 32 block of a tile: this thread's key row j against the 32
// queries qc .. qc + 31.  P = 2^(z2 - lse2) where visible, dS' = P (dP - D); P^T
// goes back to TMEM as bf16 pairs, dS'^T to shared memory.  vis_lo / vis_w: the
// visible query offsets of this row form [vis_lo, vis_lo + vis_w) (causal,
// window and streaming masks, key range); MASKED adds that test (and the keep
// bits) per element, RBF subtracts the key-norm term and sums dS' over the row.
template <bool MX, bool MASKED, bool RBF>
__device__ __forceinline__ void score_block(const BwdParams& p, const uint32_t (&sr)[32], const uint32_t (&dr)[32],
                                            const float4* __restrict__ ls4, const float4* __restrict__ ds4,
                                            int vis_lo, int vis_w, int qc, int j, float kn2, float& rowsum,
                                            uint32_t (&pk)[16], uint32_t (&dk)[16]) {
  float pr[32], dsv[32];
#pragma unroll
  for (int e4 = 0; e4 < 8; ++e4) {
    const float4 lv = ls4[e4], dv4 = ds4[e4];
    const float l2[4] = {lv.x, lv.y, lv.z, lv.w}, dd[4] = {dv4.x, dv4.y, dv4.z, dv4.w};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int e = 4 * e4 + u;
      const float nl = RBF ? -(l2[u] + kn2) : -l2[u];
      float pe = ex2(fmaf(__uint_as_float(sr[e]), p.c_z, nl));
      if constexpr (MASKED) {
        bool vis = static_cast<unsigned>(e - vis_lo) < static_cast<unsigned>(vis_w);
        if constexpr (MX) {
          // keep bit (i, j): the 32 lanes of a warp hold 32 consecutive keys, one word (broadcast)
          if (vis && p.bits != nullptr)
            vis = (__ldg(p.bits + static_cast<size_t>(qc + e) * p.words + (j >> 5)) >> (j & 31)) & 1u;
        }
        pe = vis ? pe : 0.f;
      }
      pr[e] = pe;
      dsv[e] = pe * (__uint_as_float(dr[e]) - dd[u]);
    }
  }
  if constexpr (RBF) {
#pragma unroll
    for (int e = 0; e < 32; ++e) rowsum += dsv[e];
  }
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    pk[e] = pack_bf16x2(pr[2 * e], pr[2 * e + 1]);
    dk[e] = pack_bf16x2(dsv[2 * e], dsv[2 * e + 1]);
  }
}

// MX: the streaming mask, keep bits or key padding is in use (a separate instantiation,
// so the plain masks keep their own register allocation)
template <int E, int EV, bool MX>
__global__ void __launch_bounds__(BTHREADS, 1)
    bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
               const __grid_constant__ CUtensorMap tm_dq, const BwdParams p) {
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
  volatile int* dq_issued = reinterpret_cast<volatile int*>(sp + C::OFF_MISC + 8);  // tiles whose dQ^T is issued
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
  // tile it: query head kvh * group + it / n_qt, first query (qt_lo + it % n_qt) * QT
  auto tile_q0 = [&](int it) { return (qt_lo + it % n_qt) * QT; };
  auto tile_head = [&](int it) { return (static_cast<size_t>(n) * p.Hq + kvh * p.group + it / n_qt); };

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    *dq_issued = 0;
    mbar_init(bar(C::B_KV), 1);
    for (int s = 0; s < C::NSTAGE; ++s) {
      mbar_init(bar(C::B_QFULL + s), 1);
      mbar_init(bar(C::B_QEMPTY + s), 2);  // after dP^T (dQ readout warpgroup) and after dK (second issuer)
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(C::B_SFULL + b), 2);  // S^T (second issuer) and dP^T (dQ readout warpgroup)
      mbar_init(bar(C::B_PFULL + b), N_COMPUTE);
      mbar_init(bar(C::B_DQFULL + b), 1);
    }
    mbar_init(bar(C::B_DKV), 1);
    for (int d = 0; d < 3; ++d) mbar_init(bar(C::B_DRAIN + d), 1);
    fence_barrier_init();
  }
  if (warp == W_ISSUER) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == W_PRODUCER) {
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
        const int q0 = tile_q0(it);
        const size_t head = tile_head(it);
        const int qrow = static_cast<int>(head);
        const uint32_t full = bar(C::B_QFULL + s);
        mbar_arrive_expect_tx(full, C::Q_BYTES + C::DO_BYTES + C::LD_BYTES);
        for (int b = 0; b < E / 64; ++b)
          tma_load_3d(sb + C::OFF_Q + s * C::Q_BYTES + b * (QT * 128), &tm_q, full, b * 64, q0, qrow);
        for (int b = 0; b < EV / 64; ++b)
          tma_load_3d(sb + C::OFF_DO + s * C::DO_BYTES + b * (QT * 128), &tm_do, full, b * 64, q0, qrow);
        // lse2 and D of the tile (padded rows: 256-byte aligned, inside the Lp-row head)
        const size_t pad = head * p.Lp + q0;
        bulk_load(sb + C::OFF_LD + s * C::LD_BYTES, p.lse2 + pad, QT * 4, full);
        bulk_load(sb + C::OFF_LD + s * C::LD_BYTES + QT * 4, p.dsum + pad, QT * 4, full);
        issued = it + 1;
      }
      // drain: every issued copy has landed before exit
      mbar_wait(bar(C::B_KV), 0);
      for (int it = (issued > C::NSTAGE ? issued - C::NSTAGE : 0); it < issued; ++it)
        mbar_wait(bar(C::B_QFULL + it % C::NSTAGE), (it / C::NSTAGE) & 1);
    }
  } else if (warp == W_ISSUER || warp == W_ISSUER2) {
    // ================= tcgen05 issuers =================
    // Three threads issue into the one in-order tensor pipe, so that an MMA a warpgroup waits
    // for is never held up behind another thread's blocked issue: the first issuer sends dQ^T
    // as soon as a tile's scores are consumed, the dQ readout warpgroup sends the dP^T that
    // reuses the columns it has just read, and the second issuer sends S^T, dV and dK.  A
    // commit covers its own thread's MMAs only: SFULL and QEMPTY take one commit from each of
    // their two issuers.
    if (lane == 0) {
      const bool urgent = warp == W_ISSUER;
      bool ok = bwait(bar(C::B_KV), 0, abort_flag);
      tc_fence_after();
      constexpr uint32_t hi = desc_hi_sw128(1024);
      const uint32_t k_lo_kmaj = desc_lo(sb + C::OFF_K, 16);
      const uint32_t k_lo_mn = desc_lo(sb + C::OFF_K, TB * 128);
      if (urgent) {
        // dQ^T = K^T dS'^T of tile it into DP_b once its scores are consumed (PFULL)
        for (int it = 0; ok && it < n_it; ++it) {
          const int b = it & 1;
          if (!bwait(bar(C::B_PFULL + b), (it >> 1) & 1, abort_flag)) break;
          tc_fence_after();
          const uint32_t ds_lo_mn = desc_lo(sb + C::OFF_DS + b * C::DS_BYTES, C::DS_BYTES);  // one 64-query box
#pragma unroll
          for (int kk = 0; kk < TB / 16; ++kk)
            mma_ss_h(tmem + C::T_DP + 64 * b, k_lo_mn + kk * 128, hi, ds_lo_mn + kk * 128, hi, C::IDESC_DQ,
                     kk > 0 ? 1u : 0u);
          mma_commit(bar(C::B_DQFULL + b));
          *dq_issued = it + 1;  // the second issuer's dV and dK of the tile queue behind its dQ^T
        }
      } else {
        // K-major operands step 16 along K inside 64-column boxes (of 128 key rows or 64 query rows)
        auto koff = [](int kk, int box_bytes) -> uint32_t {
          return static_cast<uint32_t>(((kk / 4) * box_bytes + (kk % 4) * 32) >> 4);
        };
        int n0 = 0, n1 = 0;  // next dV/dK, next S^T
        long long t_last = clock64();
        while (ok && n0 < n_it) {
          bool progress = false;
          // dV += P^T dO and dK += dS'^T Q of tile n0 once its scores are consumed and its dQ^T is
          // issued (its own PFULL test orders this thread after the compute warpgroups' writes)
          if (n0 < n1 && n0 < *dq_issued && mbar_test(bar(C::B_PFULL + (n0 & 1)), (n0 >> 1) & 1)) {
            tc_fence_after();
            const int b = n0 & 1, st = n0 % C::NSTAGE;
            const uint32_t do_lo_mn = desc_lo(sb + C::OFF_DO + st * C::DO_BYTES, QT * 128);
            const uint32_t q_lo_mn = desc_lo(sb + C::OFF_Q + st * C::Q_BYTES, QT * 128);
            const uint32_t ds_lo_kmaj = desc_lo(sb + C::OFF_DS + b * C::DS_BYTES, 16);
            // query q's bf16 pair of P^T sits in column 64 b + 32 (q / 32) + (q % 32) / 2
#pragma unroll
            for (int kk = 0; kk < QT / 16; ++kk)
              mma_ts_h(tmem + C::T_DV, tmem + C::T_S + 64 * b + 32 * (kk / 2) + 8 * (kk % 2), do_lo_mn + kk * 128,
                       hi, C::IDESC_DV, (n0 > 0 || kk > 0) ? 1u : 0u);
            // A = dS'^T K-major over the tile's 64 queries: 32 bytes per step
#pragma unroll
            for (int kk = 0; kk < QT / 16; ++kk)
              mma_ss_h(tmem + C::T_DK, ds_lo_kmaj + kk * 2, hi, q_lo_mn + kk * 128, hi, C::IDESC_DK,
                       (n0 > 0 || kk > 0) ? 1u : 0u);
            mma_commit(bar(C::B_QEMPTY + st));  // Q, dO, lse2 and D of this stage are no longer read here
            ++n0;
            progress = true;
          }
          // S^T = K Q^T of tile n1 into S_b once Q landed and dV of tile n1 - 2 (reading P^T there) is issued
          if (n1 < n_it && n1 - 2 < n0 && mbar_test(bar(C::B_QFULL + n1 % C::NSTAGE), (n1 / C::NSTAGE) & 1)) {
            tc_fence_after();
            const uint32_t q_lo = desc_lo(sb + C::OFF_Q + (n1 % C::NSTAGE) * C::Q_BYTES, 16);
#pragma unroll
            for (int kk = 0; kk < E / 16; ++kk)
              mma_ss_h(tmem + C::T_S + 64 * (n1 & 1), k_lo_kmaj + koff(kk, TB * 128), hi, q_lo + koff(kk, QT * 128),
                       hi, C::IDESC_S, kk > 0 ? 1u : 0u);
            mma_commit(bar(C::B_SFULL + (n1 & 1)));
            ++n1;
            progress = true;
          }
          if (progress) {
            t_last = clock64();
          } else if (*abort_flag) {
            ok = false;
          } else if (clock64() - t_last > WAIT_LIMIT_CYCLES) {
            record_timeout();
            *abort_flag = 1;
            ok = false;
          }
        }
        mma_commit(bar(C::B_DKV));  // dV and dK are this thread's
      }
      const uint32_t drain = bar(C::B_DRAIN + (urgent ? 0 : 1));
      mma_commit(drain);
      mbar_wait(drain, 0);
    }
  } else if (warp >= W_DQ) {
    // ================= dQ^T readout: lane = head-dimension index, column = query =================
    // TMEM -> registers; the elected thread then sends dP^T of tile it + 2 into the columns just
    // read (with its commits on SFULL and QEMPTY), while the warpgroup writes the tile to
    // shared memory as fp32 [query][E] for bulk tensor reduce-adds into dq (the tensor map
    // skips the rows past L).
    const int e = threadIdx.x - 32 * W_DQ;  // head-dimension index = TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const bool has_rows = (warp & 3) * 32 < E;  // lanes >= E hold nothing (E = 64)
    const bool elected = threadIdx.x == 32 * W_DQ;
    float* stage = reinterpret_cast<float*>(sp + C::OFF_DQS);
    constexpr uint32_t hi = desc_hi_sw128(1024);
    const uint32_t v_lo_kmaj = desc_lo(sb + C::OFF_V, 16);
    // dP^T = V dO^T of tile t into DP_b once its dO has landed; then this thread's reads of the stage are done
    auto issue_dp = [&](int t) -> bool {
      const int st = t % C::NSTAGE;
      if (!bwait(bar(C::B_QFULL + st), (t / C::NSTAGE) & 1, abort_flag)) return false;
      tc_fence_after();
      const uint32_t do_lo = desc_lo(sb + C::OFF_DO + st * C::DO_BYTES, 16);
#pragma unroll
      for (int kk = 0; kk < EV / 16; ++kk) {
        const uint32_t ko = static_cast<uint32_t>(((kk / 4) * (TB * 128) + (kk % 4) * 32) >> 4);
        const uint32_t kq = static_cast<uint32_t>(((kk / 4) * (QT * 128) + (kk % 4) * 32) >> 4);
        mma_ss_h(tmem + C::T_DP + 64 * (t & 1), v_lo_kmaj + ko, hi, do_lo + kq, hi, C::IDESC_S, kk > 0 ? 1u : 0u);
      }
      mma_commit(bar(C::B_SFULL + (t & 1)));
      mma_commit(bar(C::B_QEMPTY + st));
      return true;
    };
    bool issue_ok = true;  // the elected thread's own waits
    if (elected) {
      issue_ok = bwait(bar(C::B_KV), 0, abort_flag);
      for (int t = 0; issue_ok && t < 2 && t < n_it; ++t) issue_ok = issue_dp(t);
    }
    for (int it = 0; it < n_it; ++it) {
      const int b = it & 1;
      bool ready = bwait(bar(C::B_DQFULL + b), (it >> 1) & 1, abort_flag);
      tc_fence_after();
      float v[QT];
      if (has_rows && ready) {
        tmem_ld32f<0>(tmem + lane_base + C::T_DP + 64 * b, v);
        tmem_ld32f<32>(tmem + lane_base + C::T_DP + 64 * b + 32, v);
        tmem_wait_ld();
      }
      tc_fence_before();
      // every lane's loads of DP_b are complete; all four warps leave together on a failed wait
      if (!dq_bar_and(ready && issue_ok)) break;
      if (elected && it + 2 < n_it) {
        tc_fence_after();
        issue_ok = issue_dp(it + 2);
      }
      // two halves of 32 queries, each with its own bulk reduce issued by its own thread (lane 0
      // of the first and second warp: two reduces in flight): a half is rewritten once the
      // previous tile's reduce of the same half has read it
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const bool half_issuer = threadIdx.x == 32 * (W_DQ + h);
        if (half_issuer) bulk_wait_read_all();
        dq_bar();
        if (has_rows) {
#pragma unroll
          for (int c = 0; c < QT / 2; ++c) stage[(32 * h + c) * E + e] = p.c_q * v[32 * h + c];
        }
        fence_proxy_async_smem();  // the staging half is read by the bulk copy (async proxy)
        dq_bar();
        if (half_issuer) {
          bulk_reduce_add_3d(&tm_dq, sb + C::OFF_DQS + h * (QT / 2) * E * 4, 0, tile_q0(it) + 32 * h,
                             static_cast<int>(tile_head(it)));
          bulk_commit();
        }
      }
    }
    if (threadIdx.x == 32 * (W_DQ + 1)) bulk_wait_all();  // every reduce has completed before the CTA exits
    if (elected) {
      bulk_wait_all();
      mma_commit(bar(C::B_DRAIN + 2));
      mbar_wait(bar(C::B_DRAIN + 2), 0);
    }
  } else {
    // ================= compute warpgroups =================
    const int t = threadIdx.x & (TB - 1);  // TMEM lane
    const int g = threadIdx.x >> 7;        // warpgroup: queries [32 g, 32 g + 32) of each tile
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int j = k0 + t;                  // this thread's key row of S^T / dP^T
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
    // keys outside [0, S) (and, with padding, outside [ks, ke)) see no query
    const bool key_ok = j < p.S && (!MX || (j >= ks && j < ke));
    float ds_rowsum = 0.f;  // rbf: sum_i dS'_ij of this key over this warpgroup's queries
    bool ok = true;
    for (int it = 0; it < n_it; ++it) {
      const int b = it & 1, s = it % C::NSTAGE;
      const int qc = tile_q0(it) + 32 * g;  // this warpgroup's first query
      // SFULL: S^T and dP^T in TMEM; QFULL (already complete): lse2 and D of the stage are visible here
      if (!__all_sync(0xffffffffu, bwait(bar(C::B_SFULL + b), (it >> 1) & 1, abort_flag) &&
                                       bwait(bar(C::B_QFULL + s), (it / C::NSTAGE) & 1, abort_flag))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sr[32], dr[32];
      tmem_ld32(tmem + lane_base + C::T_S + 64 * b + 32 * g, sr);
      tmem_ld32(tmem + lane_base + C::T_DP + 64 * b + 32 * g, dr);
      // visible queries of this key row: [lo, hi) as offsets from qc
      const int jr = j - off - qc;  // causal: i >= j - off
      int lo = p.mask_kind != MASK_NONE ? jr : INT_MIN / 2;
      int hi = INT_MAX / 2;
      if (p.mask_kind == MASK_WINDOW) hi = jr + p.window;
      if constexpr (MX) {
        if (p.mask_kind == MASK_STREAM && j >= p.keep) hi = jr + p.window;
      }
      if (!key_ok) lo = 32;
      const int lo_c = min(max(lo, 0), 32), hi_c = min(max(hi, 0), 32);
      const int vis_w = max(hi_c - lo_c, 0);
      const bool all_vis = __all_sync(0xffffffffu, vis_w == 32) && !(MX && p.bits != nullptr);
      const float4* ls4 = reinterpret_cast<const float4*>(sp + C::OFF_LD + s * C::LD_BYTES) + 8 * g;
      const float4* ds4 = ls4 + QT / 4;
      uint32_t pk[16], dk[16];
      tmem_wait_ld();
      if (all_vis) {
        if (p.rbf)
          score_block<MX, false, true>(p, sr, dr, ls4, ds4, 0, 32, qc, j, kn2, ds_rowsum, pk, dk);
        else
          score_block<MX, false, false>(p, sr, dr, ls4, ds4, 0, 32, qc, j, kn2, ds_rowsum, pk, dk);
      } else {
        if (p.rbf)
          score_block<MX, true, true>(p, sr, dr, ls4, ds4, lo_c, vis_w, qc, j, kn2, ds_rowsum, pk, dk);
        else
          score_block<MX, true, false>(p, sr, dr, ls4, ds4, lo_c, vis_w, qc, j, kn2, ds_rowsum, pk, dk);
      }
      // P^T as bf16 pairs over S^T columns this warpgroup has already read
      tmem_st16(tmem + lane_base + C::T_S + 64 * b + 32 * g, pk);
      // dS'^T row t of buffer b: this warpgroup's queries are 16-byte units 4 g .. 4 g + 3 (SFULL
      // implies that dK and dQ^T of tile it - 2 have read the buffer)
      uint8_t* ds_row = sp + C::OFF_DS + b * C::DS_BYTES + t * 128;
#pragma unroll
      for (int v = 0; v < 4; ++v)
        *reinterpret_cast<uint4*>(ds_row + (((4 * g + v) ^ (t & 7)) << 4)) =
            make_uint4(dk[4 * v], dk[4 * v + 1], dk[4 * v + 2], dk[4 * v + 3]);
      tmem_wait_st();
      fence_proxy_async_smem();  // dS'^T is read by the tensor core (async proxy)
      tc_fence_before();
      mbar_arrive(bar(C::B_PFULL + b));
    }
    // dV (warpgroup 0) and dK (warpgroup 1) of this key row
    ok = __all_sync(0xffffffffu, ok);
    const bool grads_ready = ok && n_it > 0 && __all_sync(0xffffffffu, bwait(bar(C::B_DKV), 0, abort_flag));
    // the two warpgroups' halves of sum_i dS'_ij (rbf), exchanged through a dS'^T buffer
    // that no MMA reads any more once DKV has completed
    float* red_s = reinterpret_cast<float*>(sp + C::OFF_DS);
    if (grads_ready) red_s[g * TB + t] = ds_rowsum;
    compute_bar();
    if (grads_ready) ds_rowsum = red_s[t] + red_s[TB + t];
    float* dv_row = p.dv + (static_cast<size_t>(nh) * p.S + j) * EV;
    float* dk_row = p.dk + (static_cast<size_t>(nh) * p.S + j) * E;
    if (grads_ready) {
      tc_fence_after();
      // tcgen05.ld is warp-collective: every lane loads, only rows j < S are stored
      const bool row_ok = j < p.S;
      if (g == 0) {
#pragma unroll 1
        for (int c = 0; c < EV; c += 32) {
          uint32_t r[32];
          tmem_ld32(tmem + lane_base + C::T_DV + c, r);
          tmem_wait_ld();
          if (row_ok) {
#pragma unroll
            for (int e = 0; e < 32; e += 4)
              *reinterpret_cast<float4*>(dv_row + c + e) =
                  make_float4(__uint_as_float(r[e]), __uint_as_float(r[e + 1]), __uint_as_float(r[e + 2]),
                              __uint_as_float(r[e + 3]));
          }
        }
      } else {
        const uint8_t* kt_s = sp + C::OFF_K;
#pragma unroll 1
        for (int c = 0; c < E; c += 32) {
          uint32_t r[32];
          tmem_ld32(tmem + lane_base + C::T_DK + c, r);
          tmem_wait_ld();
          float gk[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) gk[e] = __uint_as_float(r[e]);
          if (p.rbf) {
            // - k_j * sum_i dS'_ij (k from the swizzled K tile: column c + e is 16-byte unit ((c+e)%64)/8 of box (c+e)/64)
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int cc = c + 8 * u;
              const uint4 w = *reinterpret_cast<const uint4*>(kt_s + (cc / 64) * (TB * 128) + t * 128 +
                                                              ((((cc % 64) / 8) ^ (t & 7)) << 4));
              const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                gk[8 * u + 2 * e] -= __uint_as_float(ws[e] << 16) * ds_rowsum;
                gk[8 * u + 2 * e + 1] -= __uint_as_float(ws[e] & 0xFFFF0000u) * ds_rowsum;
              }
            }
          }
          if (row_ok) {
#pragma unroll
            for (int e = 0; e < 32; e += 4)
              *reinterpret_cast<float4*>(dk_row + c + e) =
                  make_float4(p.c_q * gk[e], p.c_q * gk[e + 1], p.c_q * gk[e + 2], p.c_q * gk[e + 3]);
          }
        }
      }
    } else if (n_it == 0 && j < p.S) {
      // no query sees this key tile: its gradients are zero
      if (g == 0)
        for (int c = 0; c < EV; ++c) dv_row[c] = 0.f;
      else
        for (int c = 0; c < E; ++c) dk_row[c] = 0.f;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == W_ISSUER) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// D_i = dout_i . out_i (fp32), lse2_i = lse_i * log2e, both padded per head to Lp
// rows, and the sink gradient -sum_i 2^(s2 - lse2_i) D_i.  Past L, and on rows
// whose lse is -inf (they see no key and have no output), lse2 = +inf, so that
// 2^(z2 - lse2) = 0 there without a test; D = 0 past L.
// A row takes EV / 8 lanes, each reading 16 bytes of out and of dout; a warp covers
// 256 / EV rows of one head (Lp is a multiple of 128), so the sink gradient is
// summed over the warp before its one atomic.
template <int EV>
__global__ void __launch_bounds__(256) bwd_pre_kernel(const __nv_bfloat16* __restrict__ out,
                                                      const __nv_bfloat16* __restrict__ dout,
                                                      const float* __restrict__ lse, const float* __restrict__ sink,
                                                      float* __restrict__ dsum, float* __restrict__ lse2,
                                                      float* __restrict__ dsink, int Hq, int L, int Lp,
                                                      long long prows) {
  constexpr int LPR = EV / 8;        // lanes per row
  constexpr int RPW = 32 / LPR;      // rows per warp
  const int lane = threadIdx.x & 31;
  const long long pr = (static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5)) * RPW + lane / LPR;
  const int sub = lane % LPR;
  const bool row_in = pr < prows;
  const long long head = row_in ? pr / Lp : 0;
  const int i = row_in ? static_cast<int>(pr % Lp) : 0;
  const bool live = row_in && i < L;
  float acc = 0.f;
  if (live) {
    const long long r = head * L + i;
    const uint4 o4 = *reinterpret_cast<const uint4*>(out + r * EV + sub * 8);
    const uint4 d4 = *reinterpret_cast<const uint4*>(dout + r * EV + sub * 8);
    const uint32_t ow[4] = {o4.x, o4.y, o4.z, o4.w}, dw[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      acc = fmaf(__uint_as_float(ow[e] << 16), __uint_as_float(dw[e] << 16), acc);
      acc = fmaf(__uint_as_float(ow[e] & 0xFFFF0000u), __uint_as_float(dw[e] & 0xFFFF0000u), acc);
    }
  }
#pragma unroll
  for (int o = LPR / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  float g = 0.f;  // this row's sink-gradient term
  if (row_in && sub == 0) {
    if (!live) {
      dsum[pr] = 0.f;
      lse2[pr] = INFINITY;
    } else {
      const float l = lse[head * L + i];
      dsum[pr] = acc;
      lse2[pr] = l == -INFINITY ? INFINITY : l * LOG2E;
      if (sink != nullptr && l != -INFINITY) g = -ex2((sink[head % Hq] - l) * LOG2E) * acc;
    }
  }
  if (sink != nullptr && dsink != nullptr) {  // a caller may pass sink logits without asking for dsink
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) g += __shfl_xor_sync(0xffffffffu, g, o);
    const long long pr0 = (static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5)) * RPW;
    if (lane == 0 && pr0 < prows && g != 0.f) atomicAdd(dsink + (pr0 / Lp) % Hq, g);
  }
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// fp32 dq [heads, L, E] with an E x 32 x 1 box, no swizzle (each staging half is dense
// [32 queries][E]); reduces into rows past L are dropped by the tensor map.
bool make_map_dq(CUtensorMap* map, float* dq, int E, long long L, long long heads) {
  auto fn = reinterpret_cast<EncodeTiledFn>(tensor_map_encoder());
  if (!fn) return false;
  cuuint64_t gdim[3] = {static_cast<cuuint64_t>(E), static_cast<cuuint64_t>(L), static_cast<cuuint64_t>(heads)};
  cuuint64_t gstride[2] = {static_cast<cuuint64_t>(E) * 4, static_cast<cuuint64_t>(L) * E * 4};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(E), static_cast<cuuint32_t>(QT / 2), 1};
  cuuint32_t estride[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, dq, gdim, gstride, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
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
  constexpr long long ROWS_PER_BLOCK = 8 * (256 / EV);
  bwd_pre_kernel<EV><<<static_cast<unsigned>((prows + ROWS_PER_BLOCK - 1) / ROWS_PER_BLOCK), 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(a.out), static_cast<const __nv_bfloat16*>(a.dout), a.lse, a.sink, dsum, lse2,
      a.dsink, a.Hq, a.L, Lp, prows);
  if (cudaGetLastError() != cudaSuccess) return -13;
  CUtensorMap tq, tk, tv, tdo;
  if (!make_map_rows(&tq, a.q, E, a.L, static_cast<long long>(a.N) * a.Hq, QT)) return -13;
  if (!make_map_rows(&tdo, a.dout, EV, a.L, static_cast<long long>(a.N) * a.Hq, QT)) return -13;
  if (!make_map_rows(&tk, a.k, E, a.S, static_cast<long long>(a.N) * a.H, TB)) return -13;
  if (!make_map_rows(&tv, a.v, EV, a.S, static_cast<long long>(a.N) * a.H, TB)) return -13;
  CUtensorMap tdq;
  if (!make_map_dq(&tdq, a.dq, E, a.L, static_cast<long long>(a.N) * a.Hq)) return -13;
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
  kern<<<static_cast<unsigned>(grid), BTHREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, tdo, tdq, p);
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

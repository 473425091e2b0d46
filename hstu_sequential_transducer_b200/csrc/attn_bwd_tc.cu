// Tensor-core (tcgen05) pointwise-attention backward.
//
// For every allowed pair (i query, j key) of equation (2) of the HSTU
// walkthrough, with S = q_i.k_j + rab and A = SiLU(S)/N:
//   dA = dO_i . v_j,   dS = dA SiLU'(S) / N
//   dV_j += A dO_i,  dK_j += dS q_i,  dQ_i += dS k_j,  drab[bucket] += dS
// There is no softmax, so nothing needs row statistics: dS is elementwise.
//
// Work items are (sequence, head, 128-key tile of the history), ordered by
// descending number of query tiles and dealt round-robin to one persistent
// CTA per SM.  Per item the key tile's K and V stay in shared memory and the
// CTA walks the query tiles that see it (causal: from the key tile on;
// candidates see every history key).  The head_dim-64 kernel, on 128-query
// tiles (the head_dim-128 kernel further below walks 64-query blocks with
// its own roles):
//   warp 0      TMA producer: K, V once per item; Q_i, dO_i and the queries'
//               timestamps per query tile
//   warp 1      MMA issuer: S^T = K Q_i^T and dP^T = V dO_i^T into TMEM; then
//               dV += P^T dO_i and dK += dS^T Q_i (P^T, dS^T as TMEM A
//               operands) and dQ_i = dS K (dS from shared memory)
//   warps 2..9  two warpgroups, one key row per thread, each taking half of the
//               128 query columns: P^T and dS^T from S^T, dP^T (unscaled by
//               1/N, which the drains apply); dS into shared memory; sums of
//               dS per rab bucket; then their half of dQ_i from TMEM into the
//               fp32 dQ accumulator (vector reductions); after the last query
//               tile their half of dK, dV times SiLU'(Pre) to dPre
// TMEM (512 columns): [0,128) S^T -> P^T -> dQ_i, [128,256) dP^T -> dS^T,
// [256,384) dV, [384,512) dK.  Each warpgroup writes its P^T (dS^T) into the
// first half of its own S^T (dP^T) columns, so the two never overwrite
// values the other still reads; the dV and dK MMAs address the two
// 64-query halves of the A operand separately.
//
// As in the forward, away from the diagonal the rab bias of a key row
// against a query tile is a step function with at most two breakpoints along
// the row (time buckets are non-decreasing in the query's time), and so are
// the per-bucket sums of dS: a total and one suffix sum per breakpoint.
#include <cuda.h>

#include <type_traits>

#include "attn_sched.cuh"
#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace hstu {

using namespace tc;

namespace {

constexpr int kT = 128;
constexpr int kMaxCostB = 514;
static_assert(kMaxCostB <= kScanThreads, "one scan thread per cost bin");

struct BItem {
  int32_t b;
  int16_t kt;
  int16_t h;
};

struct BSched {
  int32_t* hist;
  int32_t* cursor;
  int32_t* total;
  BItem* items;
};

BSched bsched(void* ws) {
  BSched s;
  s.hist = static_cast<int32_t*>(ws);
  s.cursor = s.hist + kMaxCostB;
  s.total = s.cursor + kMaxCostB;
  s.items = reinterpret_cast<BItem*>(static_cast<char*>(ws) + align_up(3 * kMaxCostB * sizeof(int32_t), 256));
  return s;
}

__device__ __forceinline__ void bgeom(const AttnArgs& a, int b, int64_t& s0, int& n, int& hlen) {
  s0 = a.q_offsets[b];
  n = (int)(a.q_offsets[b + 1] - s0);
  const int m = a.num_targets ? a.num_targets[b] : 0;
  hlen = min(max(n - m, 0), n);
}

// query tiles that see key tile kt: from kt (causal) to the end
__device__ __forceinline__ int bcost(int n, int kt) { return (n + kT - 1) / kT - kt; }

__global__ void bsched_count(AttnArgs a, BSched w) {
  for (int b = blockIdx.x * blockDim.x + threadIdx.x; b < a.B; b += gridDim.x * blockDim.x) {
    int64_t s0;
    int n, hlen;
    bgeom(a, b, s0, n, hlen);
    for (int kt = 0; kt * kT < hlen; ++kt)
      atomicAdd(&w.hist[min(bcost(n, kt), kMaxCostB - 1)], a.H);
  }
}
__global__ void bsched_scan(BSched w) {
  scan_descending(w.hist, w.cursor, w.total, kMaxCostB);
}
__global__ void bsched_fill(AttnArgs a, BSched w) {
  for (int b = blockIdx.x * blockDim.x + threadIdx.x; b < a.B; b += gridDim.x * blockDim.x) {
    int64_t s0;
    int n, hlen;
    bgeom(a, b, s0, n, hlen);
    for (int kt = 0; kt * kT < hlen; ++kt) {
      const int pos = atomicAdd(&w.cursor[min(bcost(n, kt), kMaxCostB - 1)], a.H);
      for (int h = 0; h < a.H; ++h) {
        BItem it;
        it.b = b;
        it.kt = (int16_t)kt;
        it.h = (int16_t)h;
        w.items[pos + h] = it;
      }
    }
  }
}

template <int DH>
struct BCfg {
  static constexpr int BOXES = DH / 64;
  static constexpr int TILE = kT * DH * 2;          // 128 rows x DH bf16
  static constexpr int QD_BYTES = 2 * TILE;         // Q_i and dO_i
  static constexpr int TS_BYTES = kT * 8;
  static constexpr int STAGE = QD_BYTES + TS_BYTES;
  static constexpr int DS_BYTES = kT * kT * 2;      // dS [key][query] bf16
  static constexpr int SMEM_USED = 1024 + 2 * TILE + STAGE + DS_BYTES + 2048;
  // at least half of the SM's shared memory: one CTA (512 TMEM columns) per SM
  static constexpr int SMEM = SMEM_USED > 120 * 1024 ? SMEM_USED : 120 * 1024;
  static constexpr uint32_t IDESC_ST = idesc_bf16(128, kT, false, false);   // K Q^T, V dO^T
  static constexpr uint32_t IDESC_DKV = idesc_bf16(128, DH, false, true);   // P^T dO, dS^T Q
  static constexpr uint32_t IDESC_DQ = idesc_bf16(128, DH, true, true);     // dS K
};

struct BParams {
  AttnBwdArgs A;
  BSched w;
  uint32_t* status;
};

__device__ __forceinline__ float tanh_fast(float x) {
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(x));
  return t;
}

constexpr int kBThreads = 320;

constexpr int kPrefetch = 4;   // query blocks the backward producer prefetches ahead
constexpr int kActWarps = 8;

__device__ __forceinline__ int tb64(long long dt, int Bt) {
  return dt <= 0 ? 0 : min(64 - __clzll(dt), Bt - 1);
}

// Number of the 128 non-decreasing values cts[] that are <= tau.
__device__ __forceinline__ int count_le_128(const long long* cts, long long tau) {
  if (cts[127] <= tau) return 128;
  int lo = 0;
#pragma unroll
  for (int step = 64; step >= 1; step >>= 1)
    if (cts[lo + step - 1] <= tau) lo += step;
  return lo;
}

// Number of the 32 non-decreasing values cts[] that are <= tau.
__device__ __forceinline__ int count_le_32(const long long* cts, long long tau) {
  int lo = 0;
#pragma unroll
  for (int step = 16; step >= 1; step >>= 1)
    if (cts[lo + step - 1] <= tau) lo += step;
  return lo + (cts[lo] <= tau ? 1 : 0);
}

// One 32-column chunk of the fast path: h = S/2 + bias/2 where columns
// c >= p[k] add hd[k]; writes packed P and dS (unscaled) and accumulates the
// total and the per-breakpoint suffix sums of dS.
// Packed pairs of fp32 values (sm_100a f32x2 arithmetic).
__device__ __forceinline__ uint64_t f2pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

template <int NB, int E0 = 0, int NE = 32>
__device__ __forceinline__ void bwd_chunk_fast(const uint32_t (&sr)[32], const uint32_t (&dr)[32],
                                               int c0, float hb, const int (&p)[2],
                                               const float (&hd)[2], uint32_t (&pk)[16],
                                               uint32_t (&dk)[16], float& tot, float (&suf)[2]) {
  const uint64_t half2 = f2pack(0.5f, 0.5f), one2 = f2pack(1.f, 1.f), mone2 = f2pack(-1.f, -1.f);
  const uint64_t hb2 = f2pack(hb, hb);
  uint64_t tot2 = f2pack(0.f, 0.f), suf2[2] = {tot2, tot2};
#pragma unroll
  for (int e = E0; e < E0 + NE; e += 2) {
    const int c = c0 + e;
    uint64_t h = f2fma(f2pack(__uint_as_float(sr[e]), __uint_as_float(sr[e + 1])), half2, hb2);
#pragma unroll
    for (int k = 0; k < NB; ++k)
      h = f2add(h, f2pack(c >= p[k] ? hd[k] : 0.f, c + 1 >= p[k] ? hd[k] : 0.f));
    float h0, h1;
    f2unpack(h, h0, h1);
    const uint64_t t = f2pack(tanh_fast(h0), tanh_fast(h1));
    const uint64_t sg = f2fma(t, half2, half2);                  // sigmoid(x)
    const uint64_t pa = f2fma(h, t, h);                          // SiLU(x)
    const uint64_t w = f2mul(h, f2fma(t, mone2, one2));          // x (1 - sigmoid(x))
    const uint64_t ds = f2mul(f2pack(__uint_as_float(dr[e]), __uint_as_float(dr[e + 1])), f2fma(sg, w, sg));
    tot2 = f2add(tot2, ds);
    float d0, d1;
    f2unpack(ds, d0, d1);
#pragma unroll
    for (int k = 0; k < NB; ++k)
      suf2[k] = f2add(suf2[k], f2pack(c >= p[k] ? d0 : 0.f, c + 1 >= p[k] ? d1 : 0.f));
    float a0, a1;
    f2unpack(pa, a0, a1);
    pk[e / 2] = pack_bf16(a0, a1);
    dk[e / 2] = pack_bf16(d0, d1);
  }
  float x0, x1;
  f2unpack(tot2, x0, x1);
  tot += x0 + x1;
#pragma unroll
  for (int k = 0; k < NB; ++k) {
    f2unpack(suf2[k], x0, x1);
    suf[k] += x0 + x1;
  }
}

// Shared-memory float reduction issued only where pred holds (a predicated
// instruction, so per-element bucket sums need no divergent branch).
__device__ __forceinline__ void pred_red(float* addr, float v, bool pred) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %2, 0;\n\t@p red.shared.add.f32 [%0], %1;\n\t}" ::"r"(smem_u32(addr)),
      "f"(v), "r"((int)pred)
      : "memory");
}

__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b), "f"(c),
               "f"(d)
               : "memory");
}


// Byte offset of (row k, column c) in a 128-byte-swizzled MN-major tile whose
// MN extent (c) is split into 64-wide blocks `blk` bytes apart and whose K
// extent (k) runs down 128-byte rows.
__device__ __forceinline__ uint32_t mn_off(int k, int c, uint32_t blk) {
  return (uint32_t)(c >> 6) * blk + (uint32_t)(k >> 3) * 1024u + (uint32_t)(k & 7) * 128u +
         ((uint32_t)(((c & 63) >> 3) ^ (k & 7)) << 4) + (uint32_t)(c & 7) * 2u;
}

template <int DH>
__global__ void __launch_bounds__(kBThreads, 1)
    attn_bwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                       const BParams P) {
  using C = BCfg<DH>;
  // the base stays the __shared__ array itself, so that every access
  // through it compiles to a shared-memory (not a generic) access
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {              // uniform over the block: all threads leave
    if (threadIdx.x == 0 && P.status) atomicOr(P.status, kStatusSmemAlign);
    return;
  }
  uint8_t* smem = smem_raw;
  uint8_t* sK = smem;
  uint8_t* sV = sK + C::TILE;
  uint8_t* sQD = sV + C::TILE;        // Q_i | dO_i | query timestamps
  uint8_t* sDS = sQD + C::STAGE;      // dS, MN-major for the dQ MMA
  uint64_t* bars = reinterpret_cast<uint64_t*>(sDS + C::DS_BYTES);
  uint64_t* kv_full = bars + 0;
  uint64_t* kv_empty = bars + 1;
  uint64_t* qd_full = bars + 2;
  uint64_t* qd_empty = bars + 3;
  uint64_t* st_full = bars + 4;
  uint64_t* pds_full = bars + 5;
  uint64_t* dq_full = bars + 6;
  uint64_t* a_free = bars + 7;
  uint64_t* dkv_full = bars + 8;
  uint64_t* dkv_free = bars + 9;
  uint64_t* done_bar = bars + 10;
  float* rab = reinterpret_cast<float*>(bars + 12);     // [64] current head's tables
  float* drab = rab + 64;                               // [64] bucket sums of dS
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drab + 64);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const AttnArgs& a = P.A.f;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int total = *P.w.total;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 11; ++i) {
      const bool act = &bars[i] == pds_full || &bars[i] == a_free || &bars[i] == dkv_free;
      mbar_init(&bars[i], act ? kActWarps : 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tA = tmem, tB = tmem + 128, tdV = tmem + 256, tdK = tmem + 384;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    uint32_t items_done = 0, m = 0;
    bool kv_iss = false, qd_iss = false;
    uint32_t kv_par = 0, qd_par = 0;
    for (int it = blockIdx.x; it < total; it += gridDim.x) {
      if (*abort_flag) break;
      const BItem item = P.w.items[it];
      int64_t s0;
      int n, hlen;
      bgeom(a, item.b, s0, n, hlen);
      const int k0 = item.kt * kT;
      const int nqt = bcost(n, item.kt);
      bool ok = true;
      if (lane == 0) ok = mbar_wait(kv_empty, (items_done & 1) ^ 1, abort_flag, P.status);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      if (lane == 0) {
        mbar_expect_tx(kv_full, 2 * C::TILE);
#pragma unroll
        for (int x = 0; x < C::BOXES; ++x) {
          tma_load_2d(sK + x * (kT * 128), &tmK, kv_full, item.h * DH + 64 * x, (int32_t)(s0 + k0));
          tma_load_2d(sV + x * (kT * 128), &tmV, kv_full, item.h * DH + 64 * x, (int32_t)(s0 + k0));
        }
        kv_iss = true;
        kv_par = items_done & 1;
      }
      ++items_done;
      for (int qi = 0; qi < nqt; ++qi, ++m) {
        const int q0 = (item.kt + qi) * kT;
        if (lane == 0) ok = mbar_wait(qd_empty, (m & 1) ^ 1, abort_flag, P.status);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        long long* qts = reinterpret_cast<long long*>(sQD + C::QD_BYTES);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int c = lane + 32 * u;
          // past the sequence: a large sentinel keeps the staged times sorted
          qts[c] = (q0 + c < n && bounds_ok(s0 + q0 + c < a.q_rows, P.status))
                    ? a.q_ts[s0 + q0 + c] : (1LL << 62);
        }
        __syncwarp();
        if (lane == 0) {
          mbar_expect_tx(qd_full, C::QD_BYTES);
#pragma unroll
          for (int x = 0; x < C::BOXES; ++x) {
            tma_load_2d(sQD + x * (kT * 128), &tmQ, qd_full, item.h * DH + 64 * x, (int32_t)(s0 + q0));
            tma_load_2d(sQD + C::TILE + x * (kT * 128), &tmdO, qd_full, item.h * DH + 64 * x,
                        (int32_t)(s0 + q0));
          }
          qd_iss = true;
          qd_par = m & 1;
        }
      }
      if (!ok) break;
    }
    if (lane == 0) {
      volatile int never = 0;
      if (kv_iss) mbar_wait(kv_full, kv_par, &never, P.status);
      if (qd_iss) mbar_wait(qd_full, qd_par, &never, P.status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t items_done = 0, m = 0;
      const uint32_t k_s = smem_u32(sK), v_s = smem_u32(sV), qd_s = smem_u32(sQD),
                     ds_s = smem_u32(sDS);
      for (int it = blockIdx.x; it < total; it += gridDim.x) {
        if (*abort_flag) break;
        const BItem item = P.w.items[it];
        int64_t s0;
        int n, hlen;
        bgeom(a, item.b, s0, n, hlen);
        const int nqt = bcost(n, item.kt);
        if (!mbar_wait(kv_full, items_done & 1, abort_flag, P.status)) break;
        if (!mbar_wait(dkv_free, (items_done & 1) ^ 1, abort_flag, P.status)) break;
        tc_fence_after();
        bool ok = true;
        for (int qi = 0; qi < nqt; ++qi, ++m) {
          if (!mbar_wait(qd_full, m & 1, abort_flag, P.status)) { ok = false; break; }
          if (m > 0 && !mbar_wait(a_free, (m - 1) & 1, abort_flag, P.status)) { ok = false; break; }
          tc_fence_after();
          // S^T = K Q_i^T (region A), dP^T = V dO_i^T (region B)
#pragma unroll
          for (int k = 0; k < DH / 16; ++k) {
            const uint32_t off = (k / 4) * (kT * 128) + (k % 4) * 32;
            mma_ss(tA, sdesc_kmajor(k_s + off), sdesc_kmajor(qd_s + off), C::IDESC_ST, k > 0);
          }
#pragma unroll
          for (int k = 0; k < DH / 16; ++k) {
            const uint32_t off = (k / 4) * (kT * 128) + (k % 4) * 32;
            mma_ss(tB, sdesc_kmajor(v_s + off), sdesc_kmajor(qd_s + C::TILE + off), C::IDESC_ST, k > 0);
          }
          mma_commit(st_full);
          if (!mbar_wait(pds_full, m & 1, abort_flag, P.status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t acc0 = qi > 0 ? 1u : 0u;
          // dV += P^T dO_i ; dK += dS^T Q_i   (sum over the 128 queries)
          // A operand halves: queries [0,64) at columns [0,32), [64,128) at [64,96)
#pragma unroll
          for (int k = 0; k < kT / 16; ++k)
            mma_ts(tdV, tA + (k / 4) * 64 + (k % 4) * 8, sdesc_mnmajor(qd_s + C::TILE + k * 2048, kT * 128),
                   C::IDESC_DKV, (acc0 || k > 0) ? 1u : 0u);
#pragma unroll
          for (int k = 0; k < kT / 16; ++k)
            mma_ts(tdK, tB + (k / 4) * 64 + (k % 4) * 8, sdesc_mnmajor(qd_s + k * 2048, kT * 128),
                   C::IDESC_DKV, (acc0 || k > 0) ? 1u : 0u);
          // dQ_i = dS K (sum over the 128 keys) into region A
#pragma unroll
          for (int k = 0; k < kT / 16; ++k)
            mma_ss(tA, sdesc_mnmajor(ds_s + k * 2048, kT * 128), sdesc_mnmajor(k_s + k * 2048, kT * 128),
                   C::IDESC_DQ, k > 0 ? 1u : 0u);
          mma_commit(qd_empty);
          mma_commit(dq_full);
        }
        if (!ok) break;
        ++items_done;
        mma_commit(kv_empty);
        mma_commit(dkv_full);
      }
      mma_commit(done_bar);
      volatile int never = 0;
      mbar_wait(done_bar, 0, &never, P.status);
    }
  } else {
    // ------------------------------------------------------------ key-row warps
    const int quarter = warp & 3;
    const int wg = (warp - 2) >> 2;                  // query columns [64 wg, 64 wg + 64)
    const int row = quarter * 32 + lane;             // key within the tile (TMEM lane)
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    constexpr uint32_t kAct = 32 * kActWarps;
    const int d = P.A.d;
    const int odh = a.o_dh > 0 ? a.o_dh : DH;        // dQ, dPre columns stored per head
    uint32_t items_done = 0, m = 0;
    int cur_h = -1;
    const float inv_N = a.inv_N;
    const int ti = threadIdx.x - 64;                 // 0..255
    for (int it = blockIdx.x; it < total; it += gridDim.x) {
      const BItem item = P.w.items[it];
      int64_t s0;
      int n, hlen;
      bgeom(a, item.b, s0, n, hlen);
      const int k0 = item.kt * kT;
      const int nqt = bcost(n, item.kt);
      const int jk = k0 + row;                       // key index in the sequence
      const bool kvalid = jk < hlen && bounds_ok(s0 + jk < a.kv_rows, P.status);
      const long long tk = kvalid ? a.kv_ts[s0 + jk] : 0;
      if (item.h != cur_h) {
        named_barrier(1, kAct);
        if (cur_h >= 0 && ti < 64) {
          float* dst = ti < 32 ? P.A.drab_pos : P.A.drab_time;
          const int nb = ti < 32 ? a.P : a.Bt;
          const int bi = ti & 31;
          if (dst && bi < nb && drab[ti] != 0.f) atomicAdd(dst + cur_h * nb + bi, drab[ti] * inv_N);
        }
        if (ti < 32) {
          rab[ti] = (a.rab_pos && ti < a.P) ? a.rab_pos[item.h * a.P + ti] : 0.f;
          rab[32 + ti] = (a.rab_time && ti < a.Bt) ? a.rab_time[item.h * a.Bt + ti] : 0.f;
        }
        if (ti < 64) drab[ti] = 0.f;
        named_barrier(1, kAct);
        cur_h = item.h;
      }
      bool fail = *abort_flag != 0;
      if (named_barrier_any(1, kAct, fail)) break;
      const float rp_far = rab[a.P - 1];
      for (int qi = 0; qi < nqt; ++qi, ++m) {
        const int q0 = (item.kt + qi) * kT;
        fail = !mbar_wait(st_full, m & 1, abort_flag, P.status);
        if (named_barrier_any(1, kAct, fail)) { fail = true; break; }
        tc_fence_after();
        const long long* qts = reinterpret_cast<const long long*>(sQD + C::QD_BYTES);
        const int qf = q0 + wg * 64;                 // first query of this warpgroup's half
        // fast path: all 64 queries valid and causally after the key, last
        // position bucket, at most two time-bucket breakpoints
        const bool full = kvalid && qf + 63 < n && jk <= qf;
        const bool far = min(qf, hlen) - jk >= a.P - 1;
        int nb = 3, b_lo = 0;
        if (full && far) {
          b_lo = tb64(qts[wg * 64] - tk, a.Bt);
          const int b_hi = tb64(qts[wg * 64 + 63] - tk, a.Bt);
          nb = b_hi - b_lo;
        }
        const bool fast = __all_sync(0xffffffffu, full && far && nb <= 2);
        const uint32_t sA = tA + lane_off + wg * 64, sB = tB + lane_off + wg * 64;
        if (fast) {
          const int nbw = __reduce_max_sync(0xffffffffu, (unsigned)nb);
          int p[2] = {64, 64};
          float hd[2] = {0.f, 0.f};
#pragma unroll
          for (int k = 0; k < 2; ++k)
            if (k < nb) {
              const int b = b_lo + 1 + k;
              // queries with t_q - t_k >= 2^(b-1): columns c >= p
              p[k] = count_le_128(qts, tk + (1LL << (b - 1)) - 1) - wg * 64;
              hd[k] = 0.5f * (rab[32 + b] - rab[32 + b - 1]);
            }
          const float hb = 0.5f * (rp_far + rab[32 + b_lo]);
          float tot = 0.f, suf[2] = {0.f, 0.f};
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            uint32_t sr[32], dr[32], pk[16], dk[16];
            tmem_ld32(sA + c * 32, sr);
            tmem_ld32(sB + c * 32, dr);
            tmem_ld_wait();
            if (nbw == 0) bwd_chunk_fast<0>(sr, dr, c * 32, hb, p, hd, pk, dk, tot, suf);
            else if (nbw == 1) bwd_chunk_fast<1>(sr, dr, c * 32, hb, p, hd, pk, dk, tot, suf);
            else bwd_chunk_fast<2>(sr, dr, c * 32, hb, p, hd, pk, dk, tot, suf);
            tmem_st16(sA + c * 16, pk);
            tmem_st16(sB + c * 16, dk);
#pragma unroll
            for (int g8 = 0; g8 < 4; ++g8) {
              const uint4 v = make_uint4(dk[4 * g8], dk[4 * g8 + 1], dk[4 * g8 + 2], dk[4 * g8 + 3]);
              *reinterpret_cast<uint4*>(sDS + mn_off(row, wg * 64 + c * 32 + g8 * 8, kT * 128)) = v;
            }
          }
          // bucket sums: b_lo + k + 1 gets suf[k] - suf[k+1], b_lo gets tot - suf[0]
          if (kvalid) {
            atomicAdd(&drab[a.P - 1], tot);
            float below = tot;
#pragma unroll
            for (int k = 0; k < 2; ++k)
              if (k < nb) {
                atomicAdd(&drab[32 + b_lo + k], below - suf[k]);
                below = suf[k];
              }
            atomicAdd(&drab[32 + b_lo + nb], below);
          }
        } else {
          int cur_bp = -1, cur_bt = -1;
          float run_p = 0.f, run_t = 0.f;
#pragma unroll 1
          for (int c = 0; c < 2; ++c) {
            uint32_t sr[32], dr[32], pk[16], dk[16];
            tmem_ld32(sA + c * 32, sr);
            tmem_ld32(sB + c * 32, dr);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              float pv[2], dv[2];
#pragma unroll
              for (int u = 0; u < 2; ++u) {
                const int col = wg * 64 + c * 32 + e + u;
                const int qpos = q0 + col;
                const bool ok = kvalid && qpos < n && (qpos >= hlen || jk <= qpos);
                float pa = 0.f, ds = 0.f;
                if (ok) {
                  const int bp = min(max(min(qpos, hlen) - jk, 0), a.P - 1);
                  const int bt = tb64(qts[col] - tk, a.Bt);
                  const float h = 0.5f * (__uint_as_float(sr[e + u]) + rab[bp] + rab[32 + bt]);
                  const float t = tanh_fast(h);
                  const float sg = fmaf(t, 0.5f, 0.5f);
                  pa = fmaf(h, t, h);
                  ds = __uint_as_float(dr[e + u]) * fmaf(sg, fmaf(-h, t, h), sg);
                  if (bp != cur_bp) {
                    if (cur_bp >= 0) atomicAdd(&drab[cur_bp], run_p);
                    cur_bp = bp;
                    run_p = 0.f;
                  }
                  run_p += ds;
                  if (bt != cur_bt) {
                    if (cur_bt >= 0) atomicAdd(&drab[32 + cur_bt], run_t);
                    cur_bt = bt;
                    run_t = 0.f;
                  }
                  run_t += ds;
                }
                pv[u] = pa;
                dv[u] = ds;
              }
              pk[e / 2] = pack_bf16(pv[0], pv[1]);
              dk[e / 2] = pack_bf16(dv[0], dv[1]);
            }
            tmem_st16(sA + c * 16, pk);
            tmem_st16(sB + c * 16, dk);
#pragma unroll
            for (int g8 = 0; g8 < 4; ++g8) {
              const uint4 v = make_uint4(dk[4 * g8], dk[4 * g8 + 1], dk[4 * g8 + 2], dk[4 * g8 + 3]);
              *reinterpret_cast<uint4*>(sDS + mn_off(row, wg * 64 + c * 32 + g8 * 8, kT * 128)) = v;
            }
          }
          if (cur_bp >= 0) atomicAdd(&drab[cur_bp], run_p);
          if (cur_bt >= 0) atomicAdd(&drab[32 + cur_bt], run_t);
        }
        tmem_st_wait();
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(pds_full);
        // drain this warpgroup's half of dQ_i (TMEM lane = query row)
        fail = !mbar_wait(dq_full, m & 1, abort_flag, P.status);
        if (named_barrier_any(1, kAct, fail)) { fail = true; break; }
        tc_fence_after();
        const int qrow = q0 + row;
        float* dq = P.A.dq_acc + (s0 + qrow) * (int64_t)d + item.h * odh;
#pragma unroll 1
        for (int cc = 0; cc < DH / 64; ++cc) {
          const int c = wg * (DH / 64) + cc;
          if (c * 32 >= odh) continue;                 // zero-padded head columns
          uint32_t r[32];
          tmem_ld32(tA + lane_off + c * 32, r);
          tmem_ld_wait();
          if (qrow < n && bounds_ok(s0 + qrow < a.q_rows, P.status)) {
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              red_add_v4(dq + c * 32 + i, __uint_as_float(r[i]) * inv_N, __uint_as_float(r[i + 1]) * inv_N,
                         __uint_as_float(r[i + 2]) * inv_N, __uint_as_float(r[i + 3]) * inv_N);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(a_free);
      }
      if (fail) break;
      // this warpgroup's half of dK, dV (times 1/N and SiLU'(Pre)) into dPre
      fail = !mbar_wait(dkv_full, items_done & 1, abort_flag, P.status);
      ++items_done;
      if (named_barrier_any(1, kAct, fail)) break;
      tc_fence_after();
      const bf16* pre = static_cast<const bf16*>(P.A.pre);
      bf16* dpre = static_cast<bf16*>(P.A.dpre);
      const int64_t rowoff = (s0 + jk) * P.A.pre_stride;
#pragma unroll 1
      for (int cc = 0; cc < DH / 64; ++cc) {
        const int c = wg * (DH / 64) + cc;
        if (c * 32 >= odh) continue;                   // zero-padded head columns
        uint32_t rv[32], rk[32];
        tmem_ld32(tdV + lane_off + c * 32, rv);
        tmem_ld32(tdK + lane_off + c * 32, rk);
        tmem_ld_wait();
        if (kvalid) {
          const int col = item.h * odh + c * 32;
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            const uint4 pv4 = *reinterpret_cast<const uint4*>(pre + rowoff + d + col + i);
            const uint4 pk4 = *reinterpret_cast<const uint4*>(pre + rowoff + 3 * d + col + i);
            const __nv_bfloat162* pvh = reinterpret_cast<const __nv_bfloat162*>(&pv4);
            const __nv_bfloat162* pkh = reinterpret_cast<const __nv_bfloat162*>(&pk4);
            uint4 ov, ok4;
            uint32_t* ovw = reinterpret_cast<uint32_t*>(&ov);
            uint32_t* okw = reinterpret_cast<uint32_t*>(&ok4);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const float2 fv = __bfloat1622float2(pvh[u]);
              const float2 fk = __bfloat1622float2(pkh[u]);
              ovw[u] = pack_bf16(__uint_as_float(rv[i + 2 * u]) * inv_N * silu_grad_acc(fv.x),
                                 __uint_as_float(rv[i + 2 * u + 1]) * inv_N * silu_grad_acc(fv.y));
              okw[u] = pack_bf16(__uint_as_float(rk[i + 2 * u]) * inv_N * silu_grad_acc(fk.x),
                                 __uint_as_float(rk[i + 2 * u + 1]) * inv_N * silu_grad_acc(fk.y));
            }
            *reinterpret_cast<uint4*>(dpre + rowoff + d + col + i) = ov;
            *reinterpret_cast<uint4*>(dpre + rowoff + 3 * d + col + i) = ok4;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(dkv_free);
    }
    // flush the last head's bucket sums
    named_barrier(1, kAct);
    if (cur_h >= 0 && ti < 64) {
      float* dst = ti < 32 ? P.A.drab_pos : P.A.drab_time;
      const int nb = ti < 32 ? a.P : a.Bt;
      const int bi = ti & 31;
      if (dst && bi < nb && drab[ti] != 0.f) atomicAdd(dst + cur_h * nb + bi, drab[ti] * inv_N);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

int sms();

// ---------------------------------------------------------------------------
// Pipelined backward for dh = 128: 64-query blocks
// ---------------------------------------------------------------------------
// A CTA owns one (key tile, head) item at a time and walks its query blocks
// g = 0, 1, ... .  Per block the MMA thread computes S^T = K Q_g^T and
// dP^T = V dO_g^T (128 keys x 64 queries, fp32 in TMEM); the activation warps
// load both into registers and release the TMEM at once, so S^T(g+1) can be
// issued while they work.  They write P^T and dS^T (bf16 pairs) back into
// TMEM, where they are the A operands of dV += P^T dO and dK += dS^T Q, and
// dS ([key][query], a 128-byte swizzled tile) to shared memory, the
// MN-major B operand of dQ^T_g = K^T dS^T.  A warpgroup of its own drains
// dQ^T(g) from TMEM (transposes it into a dense fp32 tile in shared memory
// and adds it to the fp32 dQ accumulator with TMA bulk reduce-adds; rows past
// the sequence end carry exact zeros), so the activation warps go from one
// block to the next without it; the same warpgroup finishes an item with dK,
// dV times SiLU'(Pre) into dPre while the activation warps already work on
// the next item, whose K and V tiles the producer has prefetched into L2.
// Off the fast path, a warp whose 32 columns hold no allowed pair writes
// zeros, and time gaps within +-2^31 s take 32-bit bucket arithmetic.  Q/dO
// blocks come through a three-stage ring that the producer keeps prefetched
// into L2, so block g+1's loads overlap block g-1's dV/dK; the P^T/dS^T
// columns and the dS tile are single-buffered (block g writes them once block
// g-1's MMAs have read them).  The layout packs almost the whole 227 KB
// budget, so the kernel relies on a 1024-byte aligned dynamic shared memory
// base (checked; it reports kStatusSmemAlign if not).
// TMEM: S^T [0,64) dP^T [64,128) dQ^T [128,192) P^T [192,224) dS^T [224,256)
//       dV [256,384) dK [384,512)
constexpr int kQB = 64;
constexpr int kQStages = 3;

struct B3Cfg {
  static constexpr int DH = 128;
  static constexpr int KTILE = kT * DH * 2;            // 128 keys x 128 bf16 = 32 KB
  static constexpr int QTILE = kQB * DH * 2;           // 64 queries x 128 bf16 = 16 KB
  static constexpr int QSTAGE = 2 * QTILE;             // Q, dO
  static constexpr int TS_BYTES = kQB * 8;             // one block's times
  static constexpr int PS_BYTES = kT * kQB * 2;        // P^T or dS [key][query] for one block = 16 KB
  static constexpr int DQ_BYTES = kQB * DH * 4;        // dQ staging, 2 x [32 queries][dh] fp32 = 32 KB
  static constexpr int BAR_BYTES = 1536;               // barriers, rab tables, TMEM slot
  static constexpr int SMEM = 2 * KTILE + kQStages * QSTAGE + PS_BYTES + DQ_BYTES + kQStages * TS_BYTES +
                              BAR_BYTES;
  static constexpr uint32_t IDESC_ST = idesc_bf16(128, kQB, false, false);   // K Q^T, V dO^T
  static constexpr uint32_t IDESC_DKV = idesc_bf16(128, DH, false, true);    // P^T dO, dS^T Q
  static constexpr uint32_t IDESC_DQT = idesc_bf16(128, kQB, true, true);    // K^T dS^T
};

// query blocks that see key tile kt: from its first key to the end
__device__ __forceinline__ int qblocks(int n, int kt) { return (n - kt * kT + kQB - 1) / kQB; }

// Warp roles of the dh = 128 kernel: warpgroup 0 = producer (warp 0), MMA
// issuer (warp 1), two idle warps; warpgroups 1 and 2 = key-row warps;
// warpgroup 3 = dQ drain and the item's dK, dV epilogue.  The 65,536 registers of the launch (512 threads x
// 128) are re-split with setmaxnreg: 9,216 + 2 x 21,504 + 12,288.
constexpr int kB3Threads = 512;
constexpr int kRegCtl = 72, kRegAct = 168, kRegDrain = 96;
static_assert(128 * (kRegCtl + 2 * kRegAct + kRegDrain) <= 65536, "register split");
template <int R>
__device__ __forceinline__ void reg_dec() { asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(R)); }
template <int R>
__device__ __forceinline__ void reg_inc() { asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(R)); }

__global__ void __launch_bounds__(kB3Threads, 1)
    attn_bwd_tc3_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                        const __grid_constant__ CUtensorMap tmdQ, const BParams P) {
  using C = B3Cfg;
  static_assert(C::SMEM <= 232448, "shared memory budget");
  constexpr int DH = 128;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {              // uniform over the block: all threads leave
    if (threadIdx.x == 0 && P.status) atomicOr(P.status, kStatusSmemAlign);
    return;
  }
  uint8_t* smem = smem_raw;
  uint8_t* sK = smem;
  uint8_t* sV = sK + C::KTILE;
  uint8_t* sQD = sV + C::KTILE;                    // kQStages x (Q | dO)
  uint8_t* sDS = sQD + kQStages * C::QSTAGE;        // dS
  float* sDQ = reinterpret_cast<float*>(sDS + C::PS_BYTES);   // 2 x dQ staging [32][128]
  uint8_t* sTS = sDS + C::PS_BYTES + C::DQ_BYTES;             // kQStages x times
  uint64_t* bars = reinterpret_cast<uint64_t*>(sTS + kQStages * C::TS_BYTES);
  uint64_t* kv_full = bars + 0;
  uint64_t* kv_empty = bars + 1;
  uint64_t* qd_full = bars + 2;                     // [3] (slots 2..4)
  uint64_t* qd_empty = bars + 19;                   // [3] (slots 19..21)
  uint64_t* st_full = bars + 6;                     // S^T, dP^T of the current block are in TMEM
  uint64_t* s_free = bars + 7;                      // (8 warps) ... and have been read
  uint64_t* pds_full = bars + 8;                    // (8 warps) P^T, dS of the block are in smem
  uint64_t* ps_free = bars + 10;                    // the block's MMAs have read them
  uint64_t* dq_full = bars + 12;                    // [2] dQ^T of a block is in TMEM
  uint64_t* dq_free = bars + 14;                    // [2] (8 warps) ... and has been read
  uint64_t* dkv_full = bars + 16;
  uint64_t* dkv_free = bars + 17;                   // (8 warps)
  uint64_t* done_bar = bars + 18;
  float* rab = reinterpret_cast<float*>(bars + 24);  // [2][64] per warpgroup
  float* drab = rab + 128;                           // [2][64] per warpgroup
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drab + 128);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const AttnArgs& a = P.A.f;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int total = *P.w.total;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 22; ++i) {
      const bool act = (i == 7 || i == 8 || i == 9);
      const bool drn = (i == 14 || i == 15 || i == 17);
      mbar_init(&bars[i], act ? kActWarps : drn ? 4 : 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tD = tmem + 64;
  const uint32_t tQ = tmem + 128, tPT = tmem + 192, tDS = tmem + 224;
  const uint32_t tdV = tmem + 256, tdK = tmem + 384;

  if (warp < 4) {
  reg_dec<kRegCtl>();
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    uint32_t items_done = 0, g = 0;
    bool kv_iss = false;
    uint32_t kv_par = 0, issued = 0, issued_par = 0;
    for (int it = blockIdx.x; it < total; it += gridDim.x) {
      if (*abort_flag) break;
      const BItem item = P.w.items[it];
      int64_t s0;
      int n, hlen;
      bgeom(a, item.b, s0, n, hlen);
      const int k0 = item.kt * kT;
      const int nqb = qblocks(n, item.kt);
      bool ok = true;
      if (lane == 0) ok = mbar_wait(kv_empty, (items_done & 1) ^ 1, abort_flag, P.status);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      if (lane == 0) {
        mbar_expect_tx(kv_full, 2 * C::KTILE);
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          tma_load_2d(sK + x * (kT * 128), &tmK, kv_full, item.h * DH + 64 * x, (int32_t)(s0 + k0));
          tma_load_2d(sV + x * (kT * 128), &tmV, kv_full, item.h * DH + 64 * x, (int32_t)(s0 + k0));
        }
        kv_iss = true;
        kv_par = items_done & 1;
      }
      // the next item's K and V (they load only after this item's last MMA)
      // and its first Q/dO blocks, into L2 a few blocks before this item ends
      const int itn = it + gridDim.x;
      auto prefetch_next = [&]() {
        if (itn >= total) return;
        const BItem nx = P.w.items[itn];
        int64_t ns0;
        int nn, nhlen;
        bgeom(a, nx.b, ns0, nn, nhlen);
        const int nk0 = nx.kt * kT;
        if (lane < 4) {
          const CUtensorMap* tm = (lane & 2) ? &tmV : &tmK;
          tma_prefetch_2d(tm, nx.h * DH + 64 * (lane & 1), (int32_t)(ns0 + nk0));
        } else if (lane < 4 + 4 * kPrefetch) {
          const int mp = (lane - 4) >> 2;            // query block of the next item
          const int qp = nk0 + mp * kQB;
          if (qp < nn) {
            const CUtensorMap* tm = (lane & 2) ? &tmdO : &tmQ;
            tma_prefetch_2d(tm, nx.h * DH + 64 * (lane & 1), (int32_t)(ns0 + qp));
          }
        }
      };
      ++items_done;
      // L2 prefetch keeps the Q, dO and time rows kPrefetch blocks ahead of
      // the loads, so that a freed stage refills at L2 rather than HBM latency
      auto prefetch = [&](int mp) {
        const int qp = k0 + mp * kQB;
        if (mp >= nqb || qp >= n) return;
        if (lane < 4) {
          const CUtensorMap* tm = (lane & 2) ? &tmdO : &tmQ;
          tma_prefetch_2d(tm, item.h * DH + 64 * (lane & 1), (int32_t)(s0 + qp));
        } else if (lane < 9) {
          const int r = qp + (lane - 4) * 16;       // 16 times of 8 bytes per 128-byte line
          if (r < n && bounds_ok(s0 + r < a.q_rows, P.status)) prefetch_l2(a.q_ts + s0 + r);
        }
      };
      for (int mp = 1; mp < kPrefetch; ++mp) prefetch(mp);
      if (nqb <= kPrefetch) prefetch_next();
      for (int m = 0; m < nqb; ++m, ++g) {
        if (m == nqb - kPrefetch) prefetch_next();
        const int st = (int)(g % kQStages);
        const uint32_t par = (g / kQStages) & 1;
        const int q0 = k0 + m * kQB;
        prefetch(m + kPrefetch);
        // the block's times, read while the stage is still in use; past the
        // sequence a large sentinel keeps the staged times sorted
        long long tq[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int c = lane + 32 * u;
          tq[u] = (q0 + c < n && bounds_ok(s0 + q0 + c < a.q_rows, P.status))
                    ? a.q_ts[s0 + q0 + c] : (1LL << 62);
        }
        if (lane == 0) ok = mbar_wait(&qd_empty[st], par ^ 1, abort_flag, P.status);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        uint8_t* stg = sQD + st * C::QSTAGE;
        long long* qts = reinterpret_cast<long long*>(sTS + st * C::TS_BYTES);
        qts[lane] = tq[0];
        qts[lane + 32] = tq[1];
        __syncwarp();
        if (lane == 0) {
          mbar_expect_tx(&qd_full[st], 2 * C::QTILE);
#pragma unroll
          for (int x = 0; x < 2; ++x) {
            tma_load_2d(stg + x * (kQB * 128), &tmQ, &qd_full[st], item.h * DH + 64 * x, (int32_t)(s0 + q0));
            tma_load_2d(stg + C::QTILE + x * (kQB * 128), &tmdO, &qd_full[st], item.h * DH + 64 * x,
                        (int32_t)(s0 + q0));
          }
          issued |= 1u << st;
          issued_par = (issued_par & ~(1u << st)) | (par << st);
        }
      }
      if (!ok) break;
    }
    if (lane == 0) {
      volatile int never = 0;
      if (kv_iss) mbar_wait(kv_full, kv_par, &never, P.status);
      for (int s2 = 0; s2 < kQStages; ++s2)
        if (issued & (1u << s2)) mbar_wait(&qd_full[s2], (issued_par >> s2) & 1u, &never, P.status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t items_done = 0, g = 0;
      const uint32_t k_s = smem_u32(sK), v_s = smem_u32(sV);
      for (int it = blockIdx.x; it < total; it += gridDim.x) {
        if (*abort_flag) break;
        const BItem item = P.w.items[it];
        int64_t s0;
        int n, hlen;
        bgeom(a, item.b, s0, n, hlen);
        const int nqb = qblocks(n, item.kt);
        if (!mbar_wait(kv_full, items_done & 1, abort_flag, P.status)) break;
        tc_fence_after();
        bool ok = true;
        for (int m = 0; m <= nqb && ok; ++m) {
          if (m < nqb) {
            // block g + m: S^T, dP^T once the previous block's are in registers
            const uint32_t gb = g + m;
            const int st = (int)(gb % kQStages);
            if (!mbar_wait(&qd_full[st], (gb / kQStages) & 1, abort_flag, P.status)) { ok = false; break; }
            if (gb >= 1 && !mbar_wait(s_free, (gb - 1) & 1, abort_flag, P.status)) { ok = false; break; }
            tc_fence_after();
            const uint32_t q_s = smem_u32(sQD + st * C::QSTAGE), do_s = q_s + C::QTILE;
#pragma unroll
            for (int k = 0; k < DH / 16; ++k) {
              const uint32_t koff = (k / 4) * (kT * 128) + (k % 4) * 32;
              const uint32_t qoff = (k / 4) * (kQB * 128) + (k % 4) * 32;
              mma_ss(tS, sdesc_kmajor(k_s + koff), sdesc_kmajor(q_s + qoff), C::IDESC_ST, k > 0);
            }
#pragma unroll
            for (int k = 0; k < DH / 16; ++k) {
              const uint32_t koff = (k / 4) * (kT * 128) + (k % 4) * 32;
              const uint32_t qoff = (k / 4) * (kQB * 128) + (k % 4) * 32;
              mma_ss(tD, sdesc_kmajor(v_s + koff), sdesc_kmajor(do_s + qoff), C::IDESC_ST, k > 0);
            }
            mma_commit(st_full);
          }
          if (m >= 1) {
            // block g + m - 1: dV += P^T dO, dK += dS^T Q, dQ^T = K^T dS^T, all
            // from the P^T and dS tiles the activation warps wrote to smem
            const uint32_t gp = g + m - 1, b = gp & 1;
            const int st = (int)(gp % kQStages);
            if (m == 1 && !mbar_wait(dkv_free, (items_done & 1) ^ 1, abort_flag, P.status)) { ok = false; break; }
            if (!mbar_wait(pds_full, gp & 1, abort_flag, P.status)) { ok = false; break; }
            if (gp >= 1 && !mbar_wait(&dq_free[0], (gp - 1) & 1, abort_flag, P.status)) { ok = false; break; }
            tc_fence_after();
            const uint32_t q_s = smem_u32(sQD + st * C::QSTAGE), do_s = q_s + C::QTILE;
            const uint32_t ds_s = smem_u32(sDS);
            const uint32_t acc0 = m > 1 ? 1u : 0u;
            // A = P^T, dS^T from TMEM (16 queries = 8 packed columns per step)
#pragma unroll
            for (int k = 0; k < kQB / 16; ++k)
              mma_ts(tdV, tPT + k * 8, sdesc_mnmajor(do_s + k * 2048, kQB * 128), C::IDESC_DKV,
                     (acc0 || k > 0) ? 1u : 0u);
#pragma unroll
            for (int k = 0; k < kQB / 16; ++k)
              mma_ts(tdK, tDS + k * 8, sdesc_mnmajor(q_s + k * 2048, kQB * 128), C::IDESC_DKV,
                     (acc0 || k > 0) ? 1u : 0u);
            mma_commit(&qd_empty[st]);
#pragma unroll
            for (int k = 0; k < kT / 16; ++k)
              mma_ss(tQ, sdesc_mnmajor(k_s + k * 2048, kT * 128), sdesc_mnmajor(ds_s + k * 2048, kT * 128),
                     C::IDESC_DQT, k > 0 ? 1u : 0u);
            mma_commit(&dq_full[0]);
            mma_commit(ps_free);
          }
        }
        if (!ok) break;
        g += nqb;
        ++items_done;
        mma_commit(kv_empty);
        mma_commit(dkv_full);
      }
      mma_commit(done_bar);
      volatile int never = 0;
      mbar_wait(done_bar, 0, &never, P.status);
    }
  }
  } else if (warp >= 12) {
    // ------------------------------------------------------------ dQ drain
    reg_dec<kRegDrain>();
    // per block: dQ^T (dh rows on TMEM lanes, 64 query columns) times 1/N,
    // transposed into the staging tile, one bulk reduce-add per 32 queries
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;             // dh row (dQ^T lane)
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const int tw = threadIdx.x & 127;
    const float inv_N = a.inv_N;
    uint32_t g = 0, items_done = 0;
    bool fail = false;
    for (int it = blockIdx.x; it < total && !fail; it += gridDim.x) {
      const BItem item = P.w.items[it];
      int64_t s0;
      int n, hlen;
      bgeom(a, item.b, s0, n, hlen);
      const int k0 = item.kt * kT;
      const int nqb = qblocks(n, item.kt);
      for (int m = 0; m < nqb; ++m) {
        const uint32_t gb = g + m, b = gb & 1;
        const bool f = !mbar_wait(&dq_full[0], gb & 1, abort_flag, P.status);
        if (tw == 0) bulk_wait_read0();             // the previous block's reduces have read the staging tile
        if (named_barrier_any(4, 128, f)) { fail = true; break; }
        tc_fence_after();
        uint32_t r0[32], r1[32];
        tmem_ld32(tQ + lane_off, r0);
        tmem_ld32(tQ + lane_off + 32, r1);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&dq_free[0]);
#pragma unroll
        for (int i = 0; i < 32; ++i) sDQ[i * DH + row] = __uint_as_float(r0[i]) * inv_N;
#pragma unroll
        for (int i = 0; i < 32; ++i) sDQ[(32 + i) * DH + row] = __uint_as_float(r1[i]) * inv_N;
        fence_proxy_async_smem();
        named_barrier(4, 128);
        if (tw == 0) {
          const int32_t q = (int32_t)(s0 + k0 + m * kQB);
          tma_reduce_add_2d(&tmdQ, sDQ, item.h * DH, q);
          tma_reduce_add_2d(&tmdQ, sDQ + 32 * DH, item.h * DH, q + 32);
          bulk_commit();
        }
      }
      if (fail) break;
      g += nqb;
      // the item's dK, dV times 1/N and SiLU'(Pre) into dPre: this thread's
      // key row, 16 columns of each at a time
      if (!mbar_wait(dkv_full, items_done & 1, abort_flag, P.status)) { fail = true; break; }
      ++items_done;
      tc_fence_after();
      {
        const int jk = k0 + row;
        const bool kvalid = jk < hlen && bounds_ok(s0 + jk < a.kv_rows, P.status);
        const bf16* pre = static_cast<const bf16*>(P.A.pre);
        bf16* dpre = static_cast<bf16*>(P.A.dpre);
        const int d = P.A.d;
        const int64_t rowoff = (s0 + jk) * P.A.pre_stride;
#pragma unroll 1
        for (int c = 0; c < DH / 16; ++c) {
          uint32_t rv[16], rk[16];
          tmem_ld16(tdV + lane_off + c * 16, rv);
          tmem_ld16(tdK + lane_off + c * 16, rk);
          const int col = item.h * DH + c * 16;
          uint4 pv4[2], pk4[2];
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            pv4[i] = kvalid ? *reinterpret_cast<const uint4*>(pre + rowoff + d + col + 8 * i) : make_uint4(0, 0, 0, 0);
            pk4[i] = kvalid ? *reinterpret_cast<const uint4*>(pre + rowoff + 3 * d + col + 8 * i) : make_uint4(0, 0, 0, 0);
          }
          tmem_ld_wait();
          if (kvalid) {
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              const __nv_bfloat162* pvh = reinterpret_cast<const __nv_bfloat162*>(&pv4[i]);
              const __nv_bfloat162* pkh = reinterpret_cast<const __nv_bfloat162*>(&pk4[i]);
              uint4 ov, ok4;
              uint32_t* ovw = reinterpret_cast<uint32_t*>(&ov);
              uint32_t* okw = reinterpret_cast<uint32_t*>(&ok4);
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                const float2 fv = __bfloat1622float2(pvh[u]);
                const float2 fk = __bfloat1622float2(pkh[u]);
                const int j = 8 * i + 2 * u;
                ovw[u] = pack_bf16(__uint_as_float(rv[j]) * inv_N * silu_grad_fast(fv.x),
                                   __uint_as_float(rv[j + 1]) * inv_N * silu_grad_fast(fv.y));
                okw[u] = pack_bf16(__uint_as_float(rk[j]) * inv_N * silu_grad_fast(fk.x),
                                   __uint_as_float(rk[j + 1]) * inv_N * silu_grad_fast(fk.y));
              }
              *reinterpret_cast<uint4*>(dpre + rowoff + d + col + 8 * i) = ov;
              *reinterpret_cast<uint4*>(dpre + rowoff + 3 * d + col + 8 * i) = ok4;
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(dkv_free);
    }
    if (tw == 0) bulk_wait0();
  } else {
    // ------------------------------------------------------------ key-row warps
    reg_inc<kRegAct>();
    const int quarter = warp & 3;
    const int wg = (warp - 4) >> 2;                  // query columns [32 wg, 32 wg + 32) of a block
    const int row = quarter * 32 + lane;             // key in the tile (S^T lane) / dh row (dQ^T lane)
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    // The two warpgroups run independently: each has its own rab table, bucket
    // sums, dQ staging half and named barrier (id 2 + wg, 128 threads).
    const uint32_t bid = 2 + wg;
    float* rabw = rab + wg * 64;
    float* drabw = drab + wg * 64;
    const int d = P.A.d;
    uint32_t items_done = 0, g = 0;
    int cur_h = -1;
    const float inv_N = a.inv_N;
    const int tw = threadIdx.x & 127;                 // thread in the warpgroup
    bool fail = false;
    for (int it = blockIdx.x; it < total && !fail; it += gridDim.x) {
      const BItem item = P.w.items[it];
      int64_t s0;
      int n, hlen;
      bgeom(a, item.b, s0, n, hlen);
      const int k0 = item.kt * kT;
      const int nqb = qblocks(n, item.kt);
      const int jk = k0 + row;
      const bool kvalid = jk < hlen && bounds_ok(s0 + jk < a.kv_rows, P.status);
      const long long tk = kvalid ? a.kv_ts[s0 + jk] : 0;
      if (item.h != cur_h) {
        named_barrier(bid, 128);
        if (cur_h >= 0 && tw < 64) {
          float* dst = tw < 32 ? P.A.drab_pos : P.A.drab_time;
          const int nb = tw < 32 ? a.P : a.Bt;
          const int bi = tw & 31;
          if (dst && bi < nb && drabw[tw] != 0.f) atomicAdd(dst + cur_h * nb + bi, drabw[tw] * inv_N);
        }
        if (tw < 32) {
          rabw[tw] = (a.rab_pos && tw < a.P) ? a.rab_pos[item.h * a.P + tw] : 0.f;
          rabw[32 + tw] = (a.rab_time && tw < a.Bt) ? a.rab_time[item.h * a.Bt + tw] : 0.f;
        }
        if (tw < 64) drabw[tw] = 0.f;
        named_barrier(bid, 128);
        cur_h = item.h;
      }
      if (named_barrier_any(bid, 128, *abort_flag != 0)) { fail = true; break; }
      if (kvalid) {
        // the pre-activation lines the dK, dV epilogue reads at the item's end
        const bf16* pr = static_cast<const bf16*>(P.A.pre) + (s0 + jk) * P.A.pre_stride + item.h * DH + wg * 64;
        prefetch_l2(pr + d);
        prefetch_l2(pr + 3 * d);
      }
      const float rp_far = rabw[a.P - 1];
      // dS sums per rab bucket of this key row: the last position bucket in a
      // register, the others and the time buckets run-length encoded (both
      // buckets are non-decreasing along the row's queries), flushed to
      // shared memory only when the bucket changes and at the item's end
      float far_sum = 0.f, p_sum = 0.f, t_sum = 0.f;
      int pb_cur = -1, tb_cur = -1;
      auto add_t = [&](int bkt, float v) {
        if (bkt != tb_cur) {
          if (tb_cur >= 0) atomicAdd(&drabw[32 + tb_cur], t_sum);
          tb_cur = bkt;
          t_sum = 0.f;
        }
        t_sum += v;
      };
      auto add_p = [&](int bkt, float v) {
        if (bkt == a.P - 1) {
          far_sum += v;
          return;
        }
        if (bkt != pb_cur) {
          if (pb_cur >= 0) atomicAdd(&drabw[pb_cur], p_sum);
          pb_cur = bkt;
          p_sum = 0.f;
        }
        p_sum += v;
      };
      for (int m = 0; m < nqb; ++m) {
        const uint32_t gb = g + m, b = gb & 1;
        const int st = (int)(gb % kQStages);
        const int q0 = k0 + m * kQB;
        fail = !mbar_wait(st_full, gb & 1, abort_flag, P.status) || fail;
        tc_fence_after();
        // S^T, dP^T loads in flight while the path is chosen
        uint32_t sr[32], dr[32], pk[16], dk[16];
        tmem_ld32(tS + lane_off + wg * 32, sr);
        tmem_ld32(tD + lane_off + wg * 32, dr);
        const long long* qts = reinterpret_cast<const long long*>(sTS + st * C::TS_BYTES);
        const int qf = q0 + wg * 32;                 // first query of this warpgroup's 32
        const bool full = kvalid && qf + 31 < n && jk <= qf;
        const bool far = min(qf, hlen) - jk >= a.P - 1;
        int nb = 3, b_lo = 0;
        if (full && far) {
          b_lo = tb64(qts[wg * 32] - tk, a.Bt);
          nb = tb64(qts[wg * 32 + 31] - tk, a.Bt) - b_lo;
        }
        const bool fast = __all_sync(0xffffffffu, full && far && nb <= 1);
        // off the fast path: a warp with no allowed pair in its 32 columns
        // writes zeros; gaps within +-2^31 s take 32-bit bucket arithmetic
        const int lastc = min(31, n - 1 - qf);
        const bool any_t = kvalid && lastc >= 0 && (qf + lastc >= hlen || jk <= qf + lastc);
        bool g32_t = true;
        if (!fast && any_t) {
          const long long dlo = qts[wg * 32] - tk, dhi = qts[wg * 32 + lastc] - tk;
          g32_t = dlo > -(1LL << 31) && dhi < (1LL << 31);
        }
        const bool anyok = __any_sync(0xffffffffu, any_t);
        const bool g32 = __all_sync(0xffffffffu, g32_t);
        const uint32_t tk32 = (uint32_t)tk;
        tmem_ld_wait();
        // the scores are in registers: the next block's may overwrite them
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_free);
        // fast path: columns c >= p[k] add hd[k] to the half-bias hb
        int p[2] = {32, 32}, nbw = 0;
        float hd[2] = {0.f, 0.f}, hb = 0.f, tot = 0.f, suf[2] = {0.f, 0.f};
        if (fast) {
          nbw = __reduce_max_sync(0xffffffffu, (unsigned)nb);
#pragma unroll
          for (int k = 0; k < 2; ++k)
            if (k < nb) {
              const int bb = b_lo + 1 + k;
              // this half's queries (sorted) with t <= tk + 2^(bb-1) - 1
              p[k] = count_le_32(qts + wg * 32, tk + (1LL << (bb - 1)) - 1);
              hd[k] = 0.5f * (rabw[32 + bb] - rabw[32 + bb - 1]);
            }
          hb = 0.5f * (rp_far + rabw[32 + b_lo]);
        }
        // columns [E0, E0 + 16) of this warp's 32 (two halves keep the
        // unrolled code and its register ranges small)
        auto half = [&](auto e0c) {
          constexpr int E0 = decltype(e0c)::value;
          if (fast) {
            if (nbw == 0) bwd_chunk_fast<0, E0, 16>(sr, dr, 0, hb, p, hd, pk, dk, tot, suf);
            else bwd_chunk_fast<1, E0, 16>(sr, dr, 0, hb, p, hd, pk, dk, tot, suf);
            return;
          }
          if (!anyok) {
#pragma unroll
            for (int e = E0; e < E0 + 16; e += 2) pk[e / 2] = dk[e / 2] = 0u;
            return;
          }
          if (g32) {
#pragma unroll
            for (int e = E0; e < E0 + 16; e += 2) {
              float pv[2], dv[2];
#pragma unroll
              for (int u = 0; u < 2; ++u) {
                const int col = wg * 32 + e + u;
                const int qpos = q0 + col;
                const bool ok = kvalid && qpos < n && (qpos >= hlen || jk <= qpos);
                const int bp = min(max(min(qpos, hlen) - jk, 0), a.P - 1);
                const int dt = (int)((uint32_t)qts[col] - tk32);
                const int bt = dt <= 0 ? 0 : min(32 - __clz(dt), a.Bt - 1);
                const float h = 0.5f * (__uint_as_float(sr[e + u]) + rabw[bp] + rabw[32 + bt]);
                const float t = tanh_fast(h);
                const float sg = fmaf(t, 0.5f, 0.5f);
                const float pa = ok ? fmaf(h, t, h) : 0.f;
                const float ds = ok ? __uint_as_float(dr[e + u]) * fmaf(sg, fmaf(-h, t, h), sg) : 0.f;
                // bucket sums without branches: the position bucket straight
                // to shared memory, the time bucket run-length encoded
                const bool near = ok && bp < a.P - 1;
                pred_red(&drabw[bp], ds, near);
                far_sum += (ok && !near) ? ds : 0.f;
                const int bte = ok ? bt : tb_cur;
                const bool chg = bte != tb_cur;
                pred_red(&drabw[32 + max(tb_cur, 0)], t_sum, chg && tb_cur >= 0);
                t_sum = chg ? ds : t_sum + ds;
                tb_cur = bte;
                pv[u] = pa;
                dv[u] = ds;
              }
              pk[e / 2] = pack_bf16(pv[0], pv[1]);
              dk[e / 2] = pack_bf16(dv[0], dv[1]);
            }
            return;
          }
#pragma unroll
          for (int e = E0; e < E0 + 16; e += 2) {
            float pv[2], dv[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const int col = wg * 32 + e + u;
              const int qpos = q0 + col;
              const bool ok = kvalid && qpos < n && (qpos >= hlen || jk <= qpos);
              float pa = 0.f, ds = 0.f;
              if (ok) {
                const int bp = min(max(min(qpos, hlen) - jk, 0), a.P - 1);
                const int bt = tb64(qts[col] - tk, a.Bt);
                const float h = 0.5f * (__uint_as_float(sr[e + u]) + rabw[bp] + rabw[32 + bt]);
                const float t = tanh_fast(h);
                const float sg = fmaf(t, 0.5f, 0.5f);
                pa = fmaf(h, t, h);
                ds = __uint_as_float(dr[e + u]) * fmaf(sg, fmaf(-h, t, h), sg);
                add_p(bp, ds);
                add_t(bt, ds);
              }
              pv[u] = pa;
              dv[u] = ds;
            }
            pk[e / 2] = pack_bf16(pv[0], pv[1]);
            dk[e / 2] = pack_bf16(dv[0], dv[1]);
          }
        };
        half(std::integral_constant<int, 0>{});
        half(std::integral_constant<int, 16>{});
        if (fast) {
          far_sum += tot;
          float below = tot;
#pragma unroll
          for (int k = 0; k < 2; ++k)
            if (k < nb) {
              add_t(b_lo + k, below - suf[k]);
              below = suf[k];
            }
          add_t(b_lo + nb, below);
        }
        // P^T and dS into the tiles once block gb-1's MMAs have read them
        if (gb >= 1) fail = !mbar_wait(ps_free, (gb - 1) & 1, abort_flag, P.status) || fail;
        tc_fence_after();
        tmem_st16(tPT + lane_off + wg * 16, pk);
        tmem_st16(tDS + lane_off + wg * 16, dk);
        uint8_t* dsb = sDS;
#pragma unroll
        for (int g8 = 0; g8 < 4; ++g8) {
          const uint32_t off = mn_off(row, wg * 32 + g8 * 8, kT * 128);
          *reinterpret_cast<uint4*>(dsb + off) = make_uint4(dk[4 * g8], dk[4 * g8 + 1], dk[4 * g8 + 2], dk[4 * g8 + 3]);
        }
        tmem_st_wait();
        tc_fence_before();
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(pds_full);
      }
      // a failed wait (the kernel is aborting) ends the item loop for the
      // whole warpgroup together
      if (named_barrier_any(bid, 128, fail)) { fail = true; break; }
      // flush this key row's bucket sums
      if (tb_cur >= 0) atomicAdd(&drabw[32 + tb_cur], t_sum);
      if (pb_cur >= 0) atomicAdd(&drabw[pb_cur], p_sum);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) far_sum += __shfl_xor_sync(0xffffffffu, far_sum, o);
      if (lane == 0 && far_sum != 0.f) atomicAdd(&drabw[a.P - 1], far_sum);
      g += nqb;
    }
    // flush the last head's bucket sums
    named_barrier(bid, 128);
    if (cur_h >= 0 && tw < 64) {
      float* dst = tw < 32 ? P.A.drab_pos : P.A.drab_time;
      const int nb = tw < 32 ? a.P : a.Bt;
      const int bi = tw & 31;
      if (dst && bi < nb && drabw[tw] != 0.f) atomicAdd(dst + cur_h * nb + bi, drabw[tw] * inv_N);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

cudaError_t launch_bwd3(const AttnBwdArgs& A, void* ws, uint32_t* status, cudaStream_t s);

int sms() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

template <int DH>
cudaError_t launch_bwd(const AttnBwdArgs& A, void* ws, uint32_t* status, cudaStream_t s) {
  using C = BCfg<DH>;
  const AttnArgs& a = A.f;
  const int d = a.H * DH;
  CUtensorMap tQ, tK, tV, tdO;
  bool ok = encode_tmap_2d(&tQ, false, a.q, (uint64_t)d, (uint64_t)a.q_rows, (uint64_t)a.q_stride, 64, kT) &&
            encode_tmap_2d(&tK, false, a.k, (uint64_t)d, (uint64_t)a.kv_rows, (uint64_t)a.kv_stride, 64, kT) &&
            encode_tmap_2d(&tV, false, a.v, (uint64_t)d, (uint64_t)a.kv_rows, (uint64_t)a.kv_stride, 64, kT) &&
            encode_tmap_2d(&tdO, false, A.dout, (uint64_t)d, (uint64_t)a.q_rows, (uint64_t)a.o_stride, 64, kT);
  if (!ok) return cudaErrorInvalidValue;
  BSched w = bsched(ws);
  cudaError_t e = cudaMemsetAsync(w.hist, 0, 3 * kMaxCostB * sizeof(int32_t), s);
  if (e != cudaSuccess) return e;
  const int blocks = (a.B + 255) / 256;
  bsched_count<<<blocks, 256, 0, s>>>(a, w);
  bsched_scan<<<1, kScanThreads, 0, s>>>(w);
  bsched_fill<<<blocks, 256, 0, s>>>(a, w);
  count_launch(3);
  BParams P;
  P.A = A;
  P.w = w;
  P.status = status;
  auto kern = attn_bwd_tc_kernel<DH>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  kern<<<sms(), kBThreads, C::SMEM, s>>>(tQ, tK, tV, tdO, P);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_bwd3(const AttnBwdArgs& A, void* ws, uint32_t* status, cudaStream_t s) {
  using C = B3Cfg;
  const AttnArgs& a = A.f;
  const int d = a.H * 128;
  CUtensorMap tQ, tK, tV, tdO;
  bool ok = encode_tmap_2d(&tQ, false, a.q, (uint64_t)d, (uint64_t)a.q_rows, (uint64_t)a.q_stride, 64, kQB) &&
            encode_tmap_2d(&tK, false, a.k, (uint64_t)d, (uint64_t)a.kv_rows, (uint64_t)a.kv_stride, 64, kT) &&
            encode_tmap_2d(&tV, false, a.v, (uint64_t)d, (uint64_t)a.kv_rows, (uint64_t)a.kv_stride, 64, kT) &&
            encode_tmap_2d(&tdO, false, A.dout, (uint64_t)d, (uint64_t)a.q_rows, (uint64_t)a.o_stride, 64, kQB);
  CUtensorMap tdQ;  // fp32 [T][d] accumulator, dense 128 x 32 boxes, no swizzle
  ok = ok && encode_tmap_2d(&tdQ, true, A.dq_acc, (uint64_t)d, (uint64_t)a.q_rows, (uint64_t)A.d, 128, 32,
                            false);
  if (!ok) return cudaErrorInvalidValue;
  BSched w = bsched(ws);
  cudaError_t e = cudaMemsetAsync(w.hist, 0, 3 * kMaxCostB * sizeof(int32_t), s);
  if (e != cudaSuccess) return e;
  const int blocks = (a.B + 255) / 256;
  bsched_count<<<blocks, 256, 0, s>>>(a, w);
  bsched_scan<<<1, kScanThreads, 0, s>>>(w);
  bsched_fill<<<blocks, 256, 0, s>>>(a, w);
  count_launch(3);
  BParams P;
  P.A = A;
  P.w = w;
  P.status = status;
  e = cudaFuncSetAttribute(attn_bwd_tc3_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  attn_bwd_tc3_kernel<<<sms(), kB3Threads, C::SMEM, s>>>(tQ, tK, tV, tdO, tdQ, P);
  count_launch();
  return cudaGetLastError();
}

}  // namespace

size_t attn_bwd_sched_bytes(int B, int64_t T, int H) {
  const size_t max_items = ((size_t)(T / kT) + (size_t)B + 1) * (size_t)H;
  return align_up(3 * kMaxCostB * sizeof(int32_t), 256) + max_items * sizeof(BItem);
}

bool attention_bwd_tc_supported(int dtype, const AttnBwdArgs& A) {
  const AttnArgs& a = A.f;
  return dtype == HSTU_BF16 && (a.dh == 64 || a.dh == 128) && !a.cached && a.q_rows > 0 &&
         a.q_stride % 8 == 0 && a.kv_stride % 8 == 0 && a.o_stride % 8 == 0 && a.P <= 32 &&
         a.Bt <= 32;
}

cudaError_t attention_bwd_tc(const AttnBwdArgs& A, void* ws, uint32_t* status, cudaStream_t s) {
  if (A.f.dh == 128) return launch_bwd3(A, ws, status, s);
  return launch_bwd<64>(A, ws, status, s);
}

}  // namespace hstu

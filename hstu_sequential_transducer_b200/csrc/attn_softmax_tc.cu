// Softmax comparison attention, forward, on the tensor cores (tcgen05).
//
// The HSTU walkthrough's "No sequence-wise softmax" contrasts HSTU's
// pointwise SiLU aggregation with the softmax attention of a standard
// Transformer, and the paper's speed claim at length 8,192 (the abstract;
// the walkthrough's "The paper in 30 seconds") is against softmax
// (FlashAttention2) Transformers.  This kernel computes the softmax variant
// of equation (2) on the same score, buckets and mask,
//   O_h(i) = sum_j softmax_j(S_h(i, j)) V_h(j)   over the allowed keys j,
// with the same tiling as the pointwise kernel, so that the two can be timed
// against each other on one GPU.
//
// Work items and warp roles follow the pointwise forward: (sequence, head,
// 128-query tile) items, longest first, one persistent CTA per SM; warp 0
// loads Q and K tiles (three-stage ring) and the keys' timestamps, warp 10 V
// tiles (two stages), warp 1 issues the MMAs, warps 2..9 are two warpgroups
// that take alternate key tiles.  What differs is the online softmax:
//   * each warpgroup keeps, per query row, its own running maximum m and sum
//     l of exp2 weights over the tiles it takes, and its own O accumulator in
//     TMEM, so the two warpgroups never wait for each other's maximum;
//   * per tile: pass 1 reads S from TMEM and finds the row maximum of
//     x = (S + bias) log2(e) over allowed keys; if it exceeds the running
//     maximum by more than 8 (a factor 256), the maximum moves and the
//     warpgroup rescales its l and its O row in TMEM (O is quiescent then:
//     the tile's S was issued after the warpgroup's previous P V, and its
//     commit covers it); pass 2 reads S again and writes P = exp2(x - m) in
//     bf16 over the tile's own S columns and adds P to l;
//   * at the end of an item the two partial results (and a candidate's own
//     key, which lies outside the key tiles) are combined exactly:
//     O = sum_w 2^(m_w - M) O_w / sum_w 2^(m_w - M) l_w with M the largest m_w.
// TMEM (512 columns): S/P of warpgroup w at [128 w, 128 w + 128), O_w at
// [256 + 128 w, 256 + 128 w + DH).
#include <cuda.h>

#include "attn_sched.cuh"
#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace hstu {

using namespace tc;

namespace {

template <int DH>
struct SmxCfg {
  static constexpr int BOXES = DH / 64;
  static constexpr int TILE_BYTES = kTile * DH * 2;
  static constexpr int K_STAGES = 3;
  static constexpr int V_STAGES = 2;
  static constexpr int TS_BYTES = kTile * 8;
  static constexpr int TS_STAGES = 6;
  static constexpr int SMEM_USED = 1024 + TILE_BYTES * (1 + K_STAGES + V_STAGES) + TS_STAGES * TS_BYTES + 4096;
  static constexpr int SMEM = SMEM_USED > 120 * 1024 ? SMEM_USED : 120 * 1024;
  static constexpr uint32_t IDESC_S = idesc_bf16(128, kTile, false, false);
  static constexpr uint32_t IDESC_O = idesc_bf16(128, DH, false, true);
  static constexpr int THREADS = 352;
  static constexpr int ACT_WARPS = 8;
  static constexpr int PREFETCH = 4;
};

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleLog2 = 8.f;   // the running maximum moves only past a factor 2^8

struct SmxParams {
  AttnArgs a;
  SchedWs w;
  uint32_t* status;
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ int tb32(long long dt, int Bt) {
  return dt <= 0 ? 0 : min(64 - __clzll(dt), Bt - 1);
}

// Number of the 128 non-decreasing values cts[] that are <= tau.
__device__ __forceinline__ int le128(const long long* cts, long long tau) {
  if (cts[127] <= tau) return 128;
  int lo = 0;
#pragma unroll
  for (int step = 64; step >= 1; step >>= 1)
    if (cts[lo + step - 1] <= tau) lo += step;
  return lo;
}

// How one row sees one key tile: either a step function of the key (every
// key visible and far from the diagonal: x = S log2e + base + sum of steps[k]
// for columns c < brk[k]) or element by element.
struct TileBias {
  bool fast;
  int brk[2];
  float step[2];
  float base;
};

__device__ __forceinline__ void chunk_x(const uint32_t (&sv)[32], int c0, const TileBias& tb, bool rvalid,
                                        int k0, int kend, bool cand, int qpos, int qp_clamped, long long tq,
                                        const long long* kts, const float* rab, int P, int Bt,
                                        float (&x)[32]) {
  if (tb.fast) {
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const int c = c0 + e;
      float v = fmaf(__uint_as_float(sv[e]), kLog2e, tb.base);
      v += (c < tb.brk[0]) ? tb.step[0] : 0.f;
      v += (c < tb.brk[1]) ? tb.step[1] : 0.f;
      x[e] = v;
    }
    return;
  }
#pragma unroll
  for (int e = 0; e < 32; ++e) {
    const int c = c0 + e;
    const int jk = k0 + c;
    const bool ok = rvalid && jk < kend && (cand || jk <= qpos);
    const int bp = min(max(qp_clamped - jk, 0), P - 1);
    const int bt = tb32(tq - kts[c], Bt);
    x[e] = ok ? (__uint_as_float(sv[e]) + rab[bp] + rab[32 + bt]) * kLog2e : -INFINITY;
  }
}

template <int DH>
__global__ void __launch_bounds__(352, 1)
    attn_fwd_softmax_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                               const __grid_constant__ CUtensorMap tmV, const SmxParams P) {
  using C = SmxCfg<DH>;
  // the base stays the __shared__ array itself, so that every access
  // through it compiles to a shared-memory (not a generic) access
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {              // uniform over the block: all threads leave
    if (threadIdx.x == 0 && P.status) atomicOr(P.status, kStatusSmemAlign);
    return;
  }
  uint8_t* smem = smem_raw;
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + C::TILE_BYTES;
  uint8_t* sV = sK + C::K_STAGES * C::TILE_BYTES;
  uint8_t* sTS = sV + C::V_STAGES * C::TILE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sTS + C::TS_STAGES * C::TS_BYTES);
  uint64_t* q_full = bars;
  uint64_t* q_empty = bars + 1;
  uint64_t* k_full = bars + 2;                 // K_STAGES
  uint64_t* k_empty = k_full + C::K_STAGES;    // K_STAGES
  uint64_t* ts_free = k_empty + C::K_STAGES;   // TS_STAGES (4 warps)
  uint64_t* v_full = ts_free + C::TS_STAGES;   // V_STAGES
  uint64_t* v_empty = v_full + C::V_STAGES;    // V_STAGES
  uint64_t* s_full = v_empty + C::V_STAGES;    // 2
  uint64_t* p_full = s_full + 2;               // 2 (4 warps)
  uint64_t* o_full = p_full + 2;               // 1
  uint64_t* o_free = o_full + 1;               // 1 (8 warps)
  uint64_t* done_bar = o_free + 1;             // 1
  float* rab_all = reinterpret_cast<float*>(done_bar + 1);     // [2][64]
  float* stat = rab_all + 128;                                  // [2 warpgroups][2 (m, l)][128 rows]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(stat + 512);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const AttnArgs& a = P.a;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int total = *P.w.total;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < C::K_STAGES; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < C::TS_STAGES; ++s) mbar_init(&ts_free[s], C::ACT_WARPS / 2);
    for (int s = 0; s < C::V_STAGES; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], C::ACT_WARPS / 2);
    }
    mbar_init(o_full, 1);
    mbar_init(o_free, C::ACT_WARPS);
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  auto tS = [tmem](uint32_t w) { return tmem + w * 128u; };
  auto tO = [tmem](uint32_t w) { return tmem + 256u + w * 128u; };

  // Tile n (a running count over the CTA's items) goes to warpgroup n & 1:
  // S/P buffer n & 1 (parity (n >> 1) & 1), K stage n % K_STAGES, timestamp
  // slot n % TS_STAGES, V stage n % V_STAGES.
  if (warp == 0) {
    // ------------------------------------------------------------ K producer
    uint32_t n = 0, items_done = 0, issued = 0, issued_par = 0, q_par = 0;
    bool q_issued = false;
    for (int it = blockIdx.x; it < total; it += gridDim.x) {
      if (*abort_flag) break;
      const AttnItem item = P.w.items[it];
      const SeqGeom g = seq_geom(a, item.b);
      const int r0 = item.qt * kTile;
      const int kend = item_kend(g, item.qt);
      const int nk = (kend + kTile - 1) / kTile;
      if (nk == 0) continue;
      auto prefetch = [&](int jp) {
        if (jp >= nk) return;
        const int kp = jp * kTile;
        if (lane < C::BOXES) {
          tma_prefetch_2d(&tmK, item.h * DH + 64 * lane, (int32_t)(g.ks + kp));
        } else if (lane >= 8 && lane < 16) {
          const int r = kp + (lane - 8) * 16;
          if (r < kend) prefetch_l2(a.kv_ts + g.ks + r);
        }
      };
      for (int jp = 0; jp < C::PREFETCH; ++jp) prefetch(jp);
      bool ok = true;
      if (lane == 0) ok = mbar_wait(q_empty, (items_done & 1) ^ 1, abort_flag, P.status);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      if (lane == 0) {
        mbar_expect_tx(q_full, C::TILE_BYTES);
#pragma unroll
        for (int x = 0; x < C::BOXES; ++x)
          tma_load_2d(sQ + x * (kTile * 128), &tmQ, q_full, item.h * DH + 64 * x, (int32_t)(g.qs + r0));
        q_issued = true;
        q_par = items_done & 1;
      }
      ++items_done;
      for (int j = 0; j < nk; ++j, ++n) {
        const int stage = (int)(n % C::K_STAGES);
        const uint32_t par = (n / C::K_STAGES) & 1;
        const int k0 = j * kTile;
        prefetch(j + C::PREFETCH);
        long long tk[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int c = lane + 32 * q;
          tk[q] = (k0 + c < kend) ? a.kv_ts[g.ks + k0 + c] : (1LL << 62);
        }
        const int tslot = (int)(n % C::TS_STAGES);
        const uint32_t tpar = (n / C::TS_STAGES) & 1;
        if (lane == 0) {
          ok = mbar_wait(&k_empty[stage], par ^ 1, abort_flag, P.status);
          ok = ok && mbar_wait(&ts_free[tslot], tpar ^ 1, abort_flag, P.status);
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        long long* kts = reinterpret_cast<long long*>(sTS + tslot * C::TS_BYTES);
#pragma unroll
        for (int q = 0; q < 4; ++q) kts[lane + 32 * q] = tk[q];
        __syncwarp();
        if (lane == 0) {
          mbar_expect_tx(&k_full[stage], C::TILE_BYTES);
#pragma unroll
          for (int x = 0; x < C::BOXES; ++x)
            tma_load_2d(sK + stage * C::TILE_BYTES + x * (kTile * 128), &tmK, &k_full[stage],
                        item.h * DH + 64 * x, (int32_t)(g.ks + k0));
          issued |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (par << stage);
        }
      }
      if (!ok) break;
    }
    if (lane == 0) {
      volatile int never = 0;
      for (int s2 = 0; s2 < C::K_STAGES; ++s2)
        if (issued & (1u << s2)) mbar_wait(&k_full[s2], (issued_par >> s2) & 1u, &never, P.status);
      if (q_issued) mbar_wait(q_full, q_par, &never, P.status);
    }
  } else if (warp == 10) {
    // ------------------------------------------------------------ V producer
    uint32_t n = 0, issued = 0, issued_par = 0;
    for (int it = blockIdx.x; it < total; it += gridDim.x) {
      if (*abort_flag) break;
      const AttnItem item = P.w.items[it];
      const SeqGeom g = seq_geom(a, item.b);
      const int kend = item_kend(g, item.qt);
      const int nk = (kend + kTile - 1) / kTile;
      if (nk == 0) continue;
      auto prefetch = [&](int jp) {
        if (jp < nk && lane < C::BOXES) tma_prefetch_2d(&tmV, item.h * DH + 64 * lane, (int32_t)(g.ks + jp * kTile));
      };
      for (int jp = 0; jp < C::PREFETCH; ++jp) prefetch(jp);
      bool ok = true;
      for (int j = 0; j < nk; ++j, ++n) {
        const int stage = (int)(n % C::V_STAGES);
        const uint32_t par = (n / C::V_STAGES) & 1;
        prefetch(j + C::PREFETCH);
        if (lane == 0) ok = mbar_wait(&v_empty[stage], par ^ 1, abort_flag, P.status);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        if (lane == 0) {
          mbar_expect_tx(&v_full[stage], C::TILE_BYTES);
#pragma unroll
          for (int x = 0; x < C::BOXES; ++x)
            tma_load_2d(sV + stage * C::TILE_BYTES + x * (kTile * 128), &tmV, &v_full[stage],
                        item.h * DH + 64 * x, (int32_t)(g.ks + j * kTile));
          issued |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (par << stage);
        }
      }
      if (!ok) break;
    }
    if (lane == 0) {
      volatile int never = 0;
      for (int s2 = 0; s2 < C::V_STAGES; ++s2)
        if (issued & (1u << s2)) mbar_wait(&v_full[s2], (issued_par >> s2) & 1u, &never, P.status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t n = 0, items_done = 0;
      for (int it = blockIdx.x; it < total; it += gridDim.x) {
        if (*abort_flag) break;
        const AttnItem item = P.w.items[it];
        const SeqGeom g = seq_geom(a, item.b);
        const int kend = item_kend(g, item.qt);
        const int nk = (kend + kTile - 1) / kTile;
        if (nk == 0) continue;
        if (!mbar_wait(q_full, items_done & 1, abort_flag, P.status)) break;
        tc_fence_after();
        const uint32_t q0 = smem_u32(sQ);
        bool ok = true;
        // S runs one tile ahead of P V.  S_j overwrites buffer j & 1, whose
        // previous tile's P V was issued (and so reads its P) before.
        for (int j = 0; j <= nk; ++j) {
          if (j < nk) {
            const uint32_t nj = n + j;
            const int stage = (int)(nj % C::K_STAGES);
            if (!mbar_wait(&k_full[stage], (nj / C::K_STAGES) & 1, abort_flag, P.status)) { ok = false; break; }
            tc_fence_after();
            const uint32_t k0s = smem_u32(sK + stage * C::TILE_BYTES);
#pragma unroll
            for (int k = 0; k < DH / 16; ++k) {
              const uint32_t off = (k / 4) * (kTile * 128) + (k % 4) * 32;
              mma_ss(tS(nj & 1), sdesc_kmajor(q0 + off), sdesc_kmajor(k0s + off), C::IDESC_S, k > 0);
            }
            mma_commit(&s_full[nj & 1]);
            mma_commit(&k_empty[stage]);
            if (j == nk - 1) mma_commit(q_empty);
          }
          if (j >= 1) {
            // O_w += P_{j-1} V_{j-1}; the first tile of each warpgroup starts O_w
            const uint32_t np = n + j - 1, w = np & 1;
            if (j == 1 && !mbar_wait(o_free, (items_done & 1) ^ 1, abort_flag, P.status)) { ok = false; break; }
            const int pst = (int)(np % C::V_STAGES);
            if (!mbar_wait(&v_full[pst], (np / C::V_STAGES) & 1, abort_flag, P.status)) { ok = false; break; }
            if (!mbar_wait(&p_full[w], (np >> 1) & 1, abort_flag, P.status)) { ok = false; break; }
            tc_fence_after();
            const uint32_t v0 = smem_u32(sV + pst * C::TILE_BYTES);
            const bool first = j - 1 < 2;
#pragma unroll
            for (int k = 0; k < kTile / 16; ++k)
              mma_ts(tO(w), tS(w) + k * 8, sdesc_mnmajor(v0 + k * 2048, kTile * 128), C::IDESC_O,
                     (!first || k > 0) ? 1u : 0u);
            mma_commit(&v_empty[pst]);
          }
        }
        if (!ok) break;
        n += nk;
        ++items_done;
        mma_commit(o_full);
      }
      mma_commit(done_bar);
      volatile int never = 0;
      mbar_wait(done_bar, 0, &never, P.status);
    }
  } else if (warp < 2 + C::ACT_WARPS) {
    // ------------------------------------------------------------ softmax warpgroups
    const int quarter = warp & 3;
    const int wg = (warp - 2) >> 2;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t bid = 2 + wg;
    float* rab = rab_all + wg * 64;
    float* my_m = stat + wg * 256;          // [128] running maximum (log2 units)
    float* my_l = my_m + 128;               // [128] running sum
    uint32_t n = 0, items_done = 0;
    int cur_h = -1;
    for (int it = blockIdx.x; it < total; it += gridDim.x) {
      const AttnItem item = P.w.items[it];
      const SeqGeom g = seq_geom(a, item.b);
      const int r0 = item.qt * kTile;
      const int rows = min(kTile, g.nq - r0);
      const int kend = item_kend(g, item.qt);
      const int nk = (kend + kTile - 1) / kTile;
      const bool rvalid = row < rows;
      const int qpos = g.qbase + r0 + row;
      const int qp_clamped = min(qpos, g.hlen);
      const bool cand = qpos >= g.hlen;
      const long long tq = rvalid ? a.q_ts[g.qs + r0 + row] : 0;
      if (item.h != cur_h) {
        named_barrier(bid, 128);
        const int t = (threadIdx.x - 64) & 127;
        if (t < 32) {
          rab[t] = (a.rab_pos && t < a.P) ? a.rab_pos[item.h * a.P + t] : 0.f;
          rab[32 + t] = (a.rab_time && t < a.Bt) ? a.rab_time[item.h * a.Bt + t] : 0.f;
        }
        named_barrier(bid, 128);
        cur_h = item.h;
      }
      // every decision to stop is taken by both warpgroups together (barrier
      // 1, 256 threads), so neither is left waiting at a named barrier
      if (named_barrier_any(1, 256, *abort_flag != 0)) break;
      bool fail = false;
      float m_run = -INFINITY, l_run = 0.f;
      const float rp_far = rab[a.P - 1];
      bool started = false;                  // this warpgroup's O has a P V of this item
      for (int j = (int)((n + wg) & 1); j < nk; j += 2) {
        const uint32_t nj = n + j;
        fail = !mbar_wait(&s_full[wg], (nj >> 1) & 1, abort_flag, P.status);
        if (named_barrier_any(bid, 128, fail)) { fail = true; break; }
        tc_fence_after();
        const int kst = (int)(nj % C::TS_STAGES);
        const long long* kts = reinterpret_cast<const long long*>(sTS + kst * C::TS_BYTES);
        const int k0 = j * kTile;
        const uint32_t sbuf = tS(wg) + lane_off;
        // the bias of this row against this tile
        TileBias tb;
        tb.fast = false;
        tb.brk[0] = tb.brk[1] = 0;
        tb.step[0] = tb.step[1] = 0.f;
        tb.base = 0.f;
        {
          const bool full_tile = k0 + kTile <= kend && (cand || k0 + kTile - 1 <= qpos);
          const bool far = qp_clamped - (k0 + kTile - 1) >= a.P - 1;
          int nb = 3, b_lo = 0;
          if (rvalid && full_tile && far) {
            const int b_hi = tb32(tq - kts[0], a.Bt);
            b_lo = tb32(tq - kts[kTile - 1], a.Bt);
            nb = b_hi - b_lo;
          }
          if (rvalid && full_tile && far && nb <= 2) {
            tb.fast = true;
            tb.base = (rp_far + rab[32 + b_lo]) * kLog2e;
#pragma unroll
            for (int k = 0; k < 2; ++k)
              if (k < nb) {
                const int b = b_lo + 1 + k;
                tb.brk[k] = le128(kts, tq - (1LL << (b - 1)));
                tb.step[k] = (rab[32 + b] - rab[32 + b - 1]) * kLog2e;
              }
          }
        }
        // pass 1: the row maximum over the tile's allowed keys
        float tmax = -INFINITY;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t sv[32];
          float x[32];
          tmem_ld32(sbuf + c * 32, sv);
          tmem_ld_wait();
          chunk_x(sv, c * 32, tb, rvalid, k0, kend, cand, qpos, qp_clamped, tq, kts, rab, a.P, a.Bt, x);
#pragma unroll
          for (int e = 0; e < 32; ++e) tmax = fmaxf(tmax, x[e]);
        }
        // move the running maximum only when it grew by more than 2^8; the
        // warpgroup's O row and sum are scaled to the new maximum
        float alpha = 1.f;
        if (tmax > m_run + kRescaleLog2) {
          alpha = (m_run == -INFINITY) ? 0.f : ex2(m_run - tmax);
          m_run = tmax;
          l_run *= alpha;
        }
        if (__any_sync(0xffffffffu, alpha != 1.f) && started) {
#pragma unroll 1
          for (int c = 0; c < DH / 32; ++c) {
            uint32_t ov[32];
            tmem_ld32(tO(wg) + lane_off + c * 32, ov);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
            tmem_st16(tO(wg) + lane_off + c * 32, *reinterpret_cast<const uint32_t(*)[16]>(&ov[0]));
            tmem_st16(tO(wg) + lane_off + c * 32 + 16, *reinterpret_cast<const uint32_t(*)[16]>(&ov[16]));
          }
        }
        // pass 2: P = exp2(x - m) in bf16 over the tile's own S columns
        float lsum = 0.f;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t sv[32], pk[16];
          float x[32];
          tmem_ld32(sbuf + c * 32, sv);
          tmem_ld_wait();
          chunk_x(sv, c * 32, tb, rvalid, k0, kend, cand, qpos, qp_clamped, tq, kts, rab, a.P, a.Bt, x);
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const float p0 = x[e] == -INFINITY ? 0.f : ex2(x[e] - m_run);
            const float p1 = x[e + 1] == -INFINITY ? 0.f : ex2(x[e + 1] - m_run);
            lsum += p0 + p1;
            pk[e / 2] = pack_bf16(p0, p1);
          }
          tmem_st16(sbuf + c * 16, pk);
        }
        l_run += lsum;
        started = true;
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&p_full[wg]);
          mbar_arrive(&ts_free[kst]);
        }
      }
      n += nk;
      // ---- epilogue: combine the two warpgroups' partial softmax results
      my_m[row] = m_run;
      my_l[row] = l_run;
      if (nk > 0) {
        if (!fail) fail = !mbar_wait(o_full, items_done & 1, abort_flag, P.status);
        ++items_done;
      }
      if (named_barrier_any(1, 256, fail)) break;
      tc_fence_after();
      const float m0 = stat[row], l0 = stat[128 + row], m1 = stat[256 + row], l1 = stat[384 + row];
      const int h = item.h;
      float xs = -INFINITY;
      if (cand && rvalid) {
        // a candidate's own key is not in the key tiles
        const bf16* q = static_cast<const bf16*>(a.q) + (g.qs + r0 + row) * a.q_stride + h * DH;
        const bf16* k = static_cast<const bf16*>(a.self_k) + (g.qs + r0 + row) * a.q_stride + h * DH;
        float sdot = 0.f;
#pragma unroll 4
        for (int e = 0; e < DH; e += 8) {
          const uint4 qa = *reinterpret_cast<const uint4*>(q + e);
          const uint4 ka = *reinterpret_cast<const uint4*>(k + e);
          const __nv_bfloat162* qh = reinterpret_cast<const __nv_bfloat162*>(&qa);
          const __nv_bfloat162* kh = reinterpret_cast<const __nv_bfloat162*>(&ka);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float2 qf = __bfloat1622float2(qh[u]), kf = __bfloat1622float2(kh[u]);
            sdot = fmaf(qf.x, kf.x, sdot);
            sdot = fmaf(qf.y, kf.y, sdot);
          }
        }
        xs = (sdot + rab[0] + rab[32]) * kLog2e;
      }
      const float M = fmaxf(fmaxf(l0 > 0.f ? m0 : -INFINITY, l1 > 0.f ? m1 : -INFINITY), xs);
      const float w0 = l0 > 0.f ? ex2(m0 - M) : 0.f;
      const float w1 = l1 > 0.f ? ex2(m1 - M) : 0.f;
      const float ws = xs > -INFINITY ? ex2(xs - M) : 0.f;
      const float L = w0 * l0 + w1 * l1 + ws;
      const float inv = L > 0.f ? 1.f / L : 0.f;
      float* O = static_cast<float*>(a.o);
      const bf16* svp = static_cast<const bf16*>(a.self_v) + (g.qs + r0 + row) * a.q_stride + h * DH;
#pragma unroll 1
      for (int cc = 0; cc < DH / 64; ++cc) {
        const int c = wg * (DH / 64) + cc;
        float o[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] = 0.f;
        if (nk > 0) {
          uint32_t r0v[32], r1v[32];
          tmem_ld32(tO(0) + lane_off + c * 32, r0v);
          tmem_ld32(tO(1) + lane_off + c * 32, r1v);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            // a partial with no allowed key holds no valid TMEM values: select, not scale
            const float a0 = w0 > 0.f ? w0 * __uint_as_float(r0v[i]) : 0.f;
            const float a1 = w1 > 0.f ? w1 * __uint_as_float(r1v[i]) : 0.f;
            o[i] = a0 + a1;
          }
        }
        if (rvalid) {
          if (ws > 0.f) {
#pragma unroll
            for (int i = 0; i < 32; i += 8) {
              const uint4 va = *reinterpret_cast<const uint4*>(svp + c * 32 + i);
              const __nv_bfloat162* vh = reinterpret_cast<const __nv_bfloat162*>(&va);
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                const float2 vf = __bfloat1622float2(vh[u]);
                o[i + 2 * u] = fmaf(ws, vf.x, o[i + 2 * u]);
                o[i + 2 * u + 1] = fmaf(ws, vf.y, o[i + 2 * u + 1]);
              }
            }
          }
          float* dst = O + (g.qs + r0 + row) * a.o_stride + h * DH + c * 32;
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(dst + i) =
                make_float4(o[i] * inv, o[i + 1] * inv, o[i + 2] * inv, o[i + 3] * inv);
        }
      }
      // both warpgroups have read the statistics before either writes the next item's
      named_barrier(1, 256);
      if (nk > 0) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(o_free);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

int sm_count_smx() {
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
cudaError_t launch_smx(const AttnArgs& a, void* ws, uint32_t* status, cudaStream_t s) {
  using C = SmxCfg<DH>;
  const int d = a.H * DH;
  CUtensorMap tQ, tK, tV;
  SmxParams P;
  P.a = a;
  P.w = sched_ws(ws);
  P.status = status;
  bool ok = encode_tmap_2d(&tQ, false, a.q, (uint64_t)d, (uint64_t)a.q_rows, (uint64_t)a.q_stride, 64, kTile) &&
            encode_tmap_2d(&tK, false, a.k, (uint64_t)d, (uint64_t)a.kv_rows, (uint64_t)a.kv_stride, 64, kTile) &&
            encode_tmap_2d(&tV, false, a.v, (uint64_t)d, (uint64_t)a.kv_rows, (uint64_t)a.kv_stride, 64, kTile);
  if (!ok) return cudaErrorInvalidValue;
  cudaError_t e = build_schedule(a, ws, s);
  if (e != cudaSuccess) return e;
  auto kern = attn_fwd_softmax_tc_kernel<DH>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  kern<<<sm_count_smx(), C::THREADS, C::SMEM, s>>>(tQ, tK, tV, P);
  count_launch();
  return cudaGetLastError();
}

}  // namespace

bool softmax_fwd_tc_supported(int dtype, const AttnArgs& a) {
  return dtype == HSTU_BF16 && (a.dh == 64 || a.dh == 128) && !a.cached && a.q_rows > 0 &&
         a.kv_rows > 0 && a.q_stride % 8 == 0 && a.kv_stride % 8 == 0 && a.P <= 32 && a.Bt <= 32;
}

cudaError_t softmax_fwd_tc(const AttnArgs& a, void* ws, uint32_t* status, cudaStream_t s) {
  if (a.dh == 128) return launch_smx<128>(a, ws, status, s);
  return launch_smx<64>(a, ws, status, s);
}

}  // namespace hstu

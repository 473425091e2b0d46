// Tensor-core (tcgen05) pointwise aggregated attention, forward.
//
// Equation (2) of the HSTU walkthrough ("What an HSTU layer changes"):
//   O_h = (1/N) [M (.) SiLU(Q_h K_h^T + rab^{p,t}_h)] V_h
// with no softmax ("No sequence-wise softmax"), rab^{p,t} from relative
// position and elapsed time (course notes, "Problem 2"), the causal or
// M-FALCON target mask ("What HSTU actually changed") and ragged work
// ("Ragged kernels"): only the key tiles a query tile can see are visited.
//
// Work items are (sequence, head, 128-row query tile), ordered longest-first
// by a device-side counting sort (attn_sched) and dealt round-robin to one
// persistent CTA per SM.  Per CTA:
//   warp 0      K producer: the Q tile once per item; K tiles (128 keys) into
//               a three-stage ring, freed as soon as S = Q K^T has read the
//               tile, and the keys' timestamps into a six-slot ring of their
//               own (freed when the activation has used them)
//   warp 10     V producer: V tiles into a two-stage ring, freed by O += P V
//   warp 1      MMA issuer (one thread): S_j = Q K_j^T into one of three TMEM
//               S buffers, two tiles ahead of O += P_{j-2} V_{j-2}, which takes
//               P from TMEM (A operand in TMEM)
//   warps 2..9  two warpgroups, one query row per thread; warpgroup b takes
//               every other key tile (all 128 columns), so one warpgroup's
//               waits and bucket searches overlap the other's SiLU work: S
//               from TMEM, bucketed rab bias, mask, SiLU, P (bf16) written
//               over the first half of the tile's own S buffer; at the end of
//               an item, half of O each, times 1/N plus the candidates' self
//               term
// Both producers read timestamps ahead of their waits and keep the next
// tiles prefetched into L2, so the rings refill at L2 latency.
// TMEM (512 columns): S/P 0..2 at [128 b, 128 b + 128), O [384, 384 + DH).
// The MMAs of the one issuing thread run in issue order, so S_{j+3}, issued
// after P_j V_j, overwrites P_j only once that MMA has read it.
//
// The rab bias of one row against one key tile is cheap in the common case:
// away from the diagonal the position bucket is the last one, and the time
// bucket, a non-increasing step function of the key (timestamps are
// non-decreasing), changes at no more than two breakpoints, found by binary
// search over the tile's timestamps once per row and tile.  Rows of a warp
// that all qualify take that path (a few compares per element); the others
// (diagonal, tails, candidates' near keys) evaluate buckets per element, in a
// rolled loop over eight columns at a time (small code for a path that runs
// once or twice per item).
#include <cuda.h>

#include "attn_sched.cuh"
#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace hstu {

using namespace tc;

size_t attn_sched_bytes(int B, int64_t Tq, int H) {
  const size_t max_items = ((size_t)(Tq / kTile) + (size_t)B + 1) * (size_t)H;
  return align_up(3 * kMaxCost * sizeof(int32_t), 256) + max_items * sizeof(AttnItem);
}

SchedWs sched_ws(void* ws) {
  SchedWs s;
  s.hist = static_cast<int32_t*>(ws);
  s.cursor = s.hist + kMaxCost;
  s.total = s.cursor + kMaxCost;
  s.items = reinterpret_cast<AttnItem*>(static_cast<char*>(ws) + align_up(3 * kMaxCost * sizeof(int32_t), 256));
  return s;
}

__global__ void sched_count_kernel(AttnArgs a, SchedWs w) {
  for (int b = blockIdx.x * blockDim.x + threadIdx.x; b < a.B; b += gridDim.x * blockDim.x) {
    const SeqGeom g = seq_geom(a, b);
    const int ntile = (g.nq + kTile - 1) / kTile;
    for (int qt = 0; qt < ntile; ++qt) {
      const int cost = min((item_kend(g, qt) + kTile - 1) / kTile, kMaxCost - 1);
      atomicAdd(&w.hist[cost], a.H);
    }
  }
}

// cursor[c] = number of items of cost > c (descending order).
__global__ void sched_scan_kernel(SchedWs w) {
  scan_descending(w.hist, w.cursor, w.total, kMaxCost);
}

__global__ void sched_fill_kernel(AttnArgs a, SchedWs w) {
  for (int b = blockIdx.x * blockDim.x + threadIdx.x; b < a.B; b += gridDim.x * blockDim.x) {
    const SeqGeom g = seq_geom(a, b);
    const int ntile = (g.nq + kTile - 1) / kTile;
    for (int qt = 0; qt < ntile; ++qt) {
      const int cost = min((item_kend(g, qt) + kTile - 1) / kTile, kMaxCost - 1);
      const int pos = atomicAdd(&w.cursor[cost], a.H);
      for (int h = 0; h < a.H; ++h) {
        AttnItem it;
        it.b = b;
        it.qt = (int16_t)qt;
        it.h = (int16_t)h;
        w.items[pos + h] = it;
      }
    }
  }
}

cudaError_t build_schedule(const AttnArgs& a, void* ws, cudaStream_t s) {
  SchedWs w = sched_ws(ws);
  cudaError_t e = cudaMemsetAsync(w.hist, 0, 3 * kMaxCost * sizeof(int32_t), s);
  if (e != cudaSuccess) return e;
  const int blocks = (a.B + 255) / 256;
  sched_count_kernel<<<blocks, 256, 0, s>>>(a, w);
  sched_scan_kernel<<<1, kScanThreads, 0, s>>>(w);
  sched_fill_kernel<<<blocks, 256, 0, s>>>(a, w);
  count_launch(3);
  return cudaGetLastError();
}

namespace {

// ---------------------------------------------------------------------------
// The forward kernel
// ---------------------------------------------------------------------------
template <int DH>
struct FwdCfg {
  static constexpr int BOXES = DH / 64;                 // 64-column boxes per tile row
  static constexpr int TILE_BYTES = kTile * DH * 2;     // one 128 x DH bf16 tile
  static constexpr int K_STAGES = 3;                    // K tiles (and their timestamps)
  static constexpr int V_STAGES = 2;                    // V tiles
  static constexpr int TS_BYTES = kTile * 8;            // key timestamps of one tile
  static constexpr int TS_STAGES = 6;                   // timestamp slots (outlive the K stage)
  static constexpr int SMEM_USED = 1024 + TILE_BYTES * (1 + K_STAGES + V_STAGES) + TS_STAGES * TS_BYTES + 1024;
  // at least half of the SM's shared memory, so that one CTA (and its 512
  // TMEM columns) is resident per SM
  static constexpr int SMEM = SMEM_USED > 120 * 1024 ? SMEM_USED : 120 * 1024;
  static constexpr uint32_t IDESC_S = idesc_bf16(128, kTile, false, false);
  static constexpr uint32_t IDESC_O = idesc_bf16(128, DH, false, true);
  static constexpr uint32_t TMEM_COLS = 512;            // S/P 0..2, O
  static constexpr int THREADS = 352;                   // 11 warps (the V producer is warp 10)
  static constexpr int ACT_WARPS = 8;
  static constexpr int PREFETCH = 4;                    // key tiles kept prefetched into L2
};

struct FwdParams {
  AttnArgs a;
  SchedWs w;
  uint32_t* status;
};

// SiLU(x) from h = x / 2:  x * sigmoid(x) = h + h * tanh(h)
__device__ __forceinline__ float silu_half(float h) {
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(h));
  return fmaf(h, t, h);
}

__device__ __forceinline__ int time_bucket32(long long dt, int Bt) {
  return dt <= 0 ? 0 : min(64 - __clzll(dt), Bt - 1);
}

// Number of the 128 non-decreasing values cts[] that are <= tau.
__device__ __forceinline__ int count_le128(const long long* cts, long long tau) {
  if (cts[127] <= tau) return 128;
  int lo = 0;
#pragma unroll
  for (int step = 64; step >= 1; step >>= 1)
    if (cts[lo + step - 1] <= tau) lo += step;
  return lo;
}

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

// Activation of one 32-column chunk in the fast path: h = S/2 + bias/2 with
// the bias a step function (NB breakpoints, columns c < p[k] add hd[k]);
// returns packed bf16 SiLU values.
template <int NB>
__device__ __forceinline__ void act_chunk_fast(const uint32_t (&s)[32], int c0, float hb,
                                               const int (&p)[2], const float (&hd)[2],
                                               uint32_t (&pk)[16]) {
  const uint64_t half2 = f2pack(0.5f, 0.5f), hb2 = f2pack(hb, hb);
#pragma unroll
  for (int e = 0; e < 32; e += 2) {
    const int c = c0 + e;
    uint64_t h = f2fma(f2pack(__uint_as_float(s[e]), __uint_as_float(s[e + 1])), half2, hb2);
#pragma unroll
    for (int k = 0; k < NB; ++k)
      h = f2add(h, f2pack(c < p[k] ? hd[k] : 0.f, c + 1 < p[k] ? hd[k] : 0.f));
    float h0, h1;
    f2unpack(h, h0, h1);
    float t0, t1;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t0) : "f"(h0));
    asm("tanh.approx.f32 %0, %1;" : "=f"(t1) : "f"(h1));
    const uint64_t y = f2fma(h, f2pack(t0, t1), h);     // SiLU = h + h tanh(h)
    float y0, y1;
    f2unpack(y, y0, y1);
    pk[e / 2] = pack_bf16(y0, y1);
  }
}

// The fast path over a whole 128-column tile, 32 columns at a time (the
// other warpgroup's work covers the TMEM load latency).
template <int NB>
__device__ __forceinline__ void act_tile_fast(uint32_t sbuf, uint32_t pbuf, float hb, const int (&p)[2],
                                              const float (&hd)[2]) {
#pragma unroll 1
  for (int c = 0; c < 4; ++c) {
    uint32_t sv[32], pk[16];
    tmem_ld32(sbuf + c * 32, sv);
    tmem_ld_wait();
    act_chunk_fast<NB>(sv, c * 32, hb, p, hd, pk);
    tmem_st16(pbuf + c * 16, pk);
  }
}

template <int DH>
__global__ void __launch_bounds__(352, 1)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const FwdParams P) {
  using C = FwdCfg<DH>;
  // the base stays the __shared__ array itself, so that every access
  // through it compiles to a shared-memory (not a generic) access
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {              // uniform over the block: all threads leave
    if (threadIdx.x == 0 && P.status) atomicOr(P.status, kStatusSmemAlign);
    return;
  }
  uint8_t* smem = smem_raw;
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + C::TILE_BYTES;                      // K_STAGES tiles
  uint8_t* sV = sK + C::K_STAGES * C::TILE_BYTES;        // V_STAGES tiles
  uint8_t* sTS = sV + C::V_STAGES * C::TILE_BYTES;       // K_STAGES x timestamps
  uint64_t* bars = reinterpret_cast<uint64_t*>(sTS + C::TS_STAGES * C::TS_BYTES);
  uint64_t* q_full = bars;                   // 1
  uint64_t* q_empty = bars + 1;              // 1
  uint64_t* k_full = bars + 2;               // K_STAGES
  uint64_t* k_empty = k_full + C::K_STAGES;  // K_STAGES: S has read the K tile
  uint64_t* ts_free = k_empty + C::K_STAGES; // TS_STAGES (4 warps): the tile's timestamps are read
  uint64_t* v_full = ts_free + C::TS_STAGES; // V_STAGES
  uint64_t* v_empty = v_full + C::V_STAGES;  // V_STAGES
  uint64_t* s_full = v_empty + C::V_STAGES;  // 3
  uint64_t* p_full = s_full + 3;             // 3
  uint64_t* o_full = p_full + 3;             // 1
  uint64_t* o_free = o_full + 1;             // 1
  uint64_t* done_bar = o_free + 1;           // 1
  float* rab_all = reinterpret_cast<float*>(done_bar + 1);   // per warpgroup [2][32] of its head
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(rab_all + 128);
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
    for (int s = 0; s < C::TS_STAGES; ++s) mbar_init(&ts_free[s], C::ACT_WARPS / 2);   // the warpgroup that took the tile
    for (int s = 0; s < C::V_STAGES; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int i = 0; i < 3; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], C::ACT_WARPS / 2);       // the warpgroup of the tile in buffer i
    }
    mbar_init(o_full, 1);
    mbar_init(o_free, C::ACT_WARPS);
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, C::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // S buffer b at columns [128 b, 128 b + 128) (b < 3); P of the tile is
  // written over the first 64 columns of its own S buffer (bf16 pairs), chunk
  // c over S columns [16 c, 16 c + 16), which chunk c / 2 <= c has already
  // loaded; O at [384, 384 + DH)
  auto tS = [tmem](uint32_t b) { return tmem + b * 128u; };
  const uint32_t tO = tmem + 384;
  auto tP = [tmem](uint32_t b) { return tmem + b * 128u; };

  // Every role walks the same item sequence and numbers the key tiles it
  // meets with one running counter n: K stage n % K_STAGES (parity
  // (n / K_STAGES) & 1), timestamp slot n % TS_STAGES, V stage n % V_STAGES,
  // S/P buffer n % 3 (parity (n / 3) & 1); warpgroup n & 1 takes tile n.
  if (warp == 0) {
    // ------------------------------------------------------------ K producer
    uint32_t n = 0, items_done = 0;
    uint32_t issued = 0, issued_par = 0;
    bool q_issued = false;
    uint32_t q_par = 0;
    for (int it = blockIdx.x; it < total; it += gridDim.x) {
      if (*abort_flag) break;
      const AttnItem item = P.w.items[it];
      const SeqGeom g = seq_geom(a, item.b);
      const int r0 = item.qt * kTile;
      const int kend = item_kend(g, item.qt);
      const int nk = (kend + kTile - 1) / kTile;
      if (nk == 0) continue;
      // L2 prefetch of key tile jp: K rows and their timestamps
      auto prefetch = [&](int jp) {
        if (jp >= nk) return;
        const int kp = jp * kTile;
        if (lane < C::BOXES) {
          tma_prefetch_2d(&tmK, item.h * DH + 64 * lane, (int32_t)(g.ks + kp));
        } else if (lane >= 8 && lane < 16) {
          const int r = kp + (lane - 8) * 16;          // 16 times per 128-byte line
          if (r < kend && bounds_ok(g.ks + r < a.kv_rows, P.status)) prefetch_l2(a.kv_ts + g.ks + r);
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
        // the tile's times, read while the stage is still in use; past the
        // visible keys a large sentinel keeps the staged times sorted
        long long tk[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int c = lane + 32 * q;
          tk[q] = (k0 + c < kend && bounds_ok(g.ks + k0 + c < a.kv_rows, P.status))
                      ? a.kv_ts[g.ks + k0 + c] : (1LL << 62);
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
        // S runs two tiles ahead of P V: S_j goes to buffer (n + j) % 3, whose
        // previous tile's P V was issued (and its P read) before
        for (int j = 0; j <= nk + 1; ++j) {
          if (j < nk) {
            const uint32_t nj = n + j;
            const int stage = (int)(nj % C::K_STAGES);
            if (!mbar_wait(&k_full[stage], (nj / C::K_STAGES) & 1, abort_flag, P.status)) { ok = false; break; }
            tc_fence_after();
            // descriptors built once per tile; a K step moves only the start
            // address field (bits 0..13, address / 16), which cannot carry
            const uint64_t qd = sdesc_kmajor(q0);
            const uint64_t kd = sdesc_kmajor(smem_u32(sK + stage * C::TILE_BYTES));
#pragma unroll
            for (int k = 0; k < DH / 16; ++k) {
              const uint32_t off = ((k / 4) * (kTile * 128) + (k % 4) * 32) >> 4;
              mma_ss(tS(nj % 3), qd + off, kd + off, C::IDESC_S, k > 0);
            }
            mma_commit(&s_full[nj % 3]);
            mma_commit(&k_empty[stage]);
            if (j == nk - 1) mma_commit(q_empty);
          }
          if (j >= 2) {
            // O += P_{j-2} V_{j-2}
            const uint32_t np = n + j - 2;
            if (j == 2 && !mbar_wait(o_free, (items_done & 1) ^ 1, abort_flag, P.status)) { ok = false; break; }
            const int pst = (int)(np % C::V_STAGES);
            if (!mbar_wait(&v_full[pst], (np / C::V_STAGES) & 1, abort_flag, P.status)) { ok = false; break; }
            if (!mbar_wait(&p_full[np % 3], (np / 3) & 1, abort_flag, P.status)) { ok = false; break; }
            tc_fence_after();
            const uint64_t vd = sdesc_mnmajor(smem_u32(sV + pst * C::TILE_BYTES), kTile * 128);
#pragma unroll
            for (int k = 0; k < kTile / 16; ++k)
              mma_ts(tO, tP(np % 3) + k * 8, vd + (uint64_t)(k * 2048 >> 4), C::IDESC_O,
                     (j > 2 || k > 0) ? 1u : 0u);
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
    // ------------------------------------------------------------ activation + epilogue
    const int quarter = warp & 3;
    const int wg = (warp - 2) >> 2;                 // takes the tiles of buffer wg; O columns [DH/2 wg, ...)
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t bid = 2 + wg;                    // this warpgroup's named barrier (128 threads)
    float* rab = rab_all + wg * 64;
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
      // rows of the query tensor this thread reads and writes directly
      const bool row_in = !rvalid || bounds_ok(g.qs + r0 + row < a.q_rows, P.status);
      const long long tq = rvalid && row_in ? a.q_ts[g.qs + r0 + row] : 0;
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
      bool stop = *abort_flag != 0;
      if (named_barrier_any(bid, 128, stop)) break;
      bool fail = false;
      const float rp_far = rab[a.P - 1];
      for (int j = (int)((n + wg) & 1); j < nk; j += 2) {   // the tiles of buffer wg
        const uint32_t nj = n + j;
        const uint32_t buf = nj % 3, par = (nj / 3) & 1;
        fail = !mbar_wait(&s_full[buf], par, abort_flag, P.status);
        if (named_barrier_any(bid, 128, fail)) { fail = true; break; }
        tc_fence_after();
        const int kst = (int)(nj % C::TS_STAGES);
        const long long* kts = reinterpret_cast<const long long*>(sTS + kst * C::TS_BYTES);
        const int k0 = j * kTile;
        // fast path: every key of the tile visible, last position bucket,
        // at most two time-bucket breakpoints along the row
        const bool full_tile = k0 + kTile <= kend && (cand || k0 + kTile - 1 <= qpos);
        const bool far = qp_clamped - (k0 + kTile - 1) >= a.P - 1;
        int nb = 3, b_lo = 0;
        if (rvalid && full_tile && far) {
          const int b_hi = time_bucket32(tq - kts[0], a.Bt);
          b_lo = time_bucket32(tq - kts[kTile - 1], a.Bt);
          nb = b_hi - b_lo;
        }
        const bool fast = __all_sync(0xffffffffu, rvalid && full_tile && far && nb <= 2);
        const uint32_t sbuf = tS(buf) + lane_off;
        const uint32_t pbuf = tP(buf) + lane_off;
        if (fast) {
          const int nbw = __reduce_max_sync(0xffffffffu, (unsigned)nb);
          int p[2] = {0, 0};
          float hd[2] = {0.f, 0.f};
#pragma unroll
          for (int k = 0; k < 2; ++k)
            if (k < nb) {
              const int b = b_lo + 1 + k;
              p[k] = count_le128(kts, tq - (1LL << (b - 1)));
              hd[k] = 0.5f * (rab[32 + b] - rab[32 + b - 1]);
            }
          const float hb = 0.5f * (rp_far + rab[32 + b_lo]);
          if (nbw == 0) act_tile_fast<0>(sbuf, pbuf, hb, p, hd);
          else if (nbw == 1) act_tile_fast<1>(sbuf, pbuf, hb, p, hd);
          else act_tile_fast<2>(sbuf, pbuf, hb, p, hd);
        } else {
          // diagonal, partial and near tiles, once or twice per item: every
          // element on its own, eight columns per pass of a rolled loop.  The
          // code stays small, so that between two such tiles the fast path
          // does not push it out of the instruction cache.
#pragma unroll 1
          for (int c8 = 0; c8 < kTile / 8; ++c8) {
            const int col0 = c8 * 8;
            uint32_t sv[8], pk[4];
            tmem_ld8(sbuf + col0, sv);
            const int j0 = k0 + col0;
            const bool all_masked = __all_sync(0xffffffffu, !rvalid || j0 >= kend || (!cand && j0 > qpos));
            tmem_ld_wait();
            if (all_masked) {
#pragma unroll
              for (int e = 0; e < 4; ++e) pk[e] = 0u;
            } else {
#pragma unroll
              for (int e = 0; e < 8; e += 2) {
                float y[2];
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                  const int jk = j0 + e + u;
                  const bool ok = rvalid && jk < kend && (cand || jk <= qpos);
                  const int bp = min(max(qp_clamped - jk, 0), a.P - 1);
                  const int bt = time_bucket32(tq - kts[col0 + e + u], a.Bt);
                  const float h = 0.5f * (__uint_as_float(sv[e + u]) + rab[bp] + rab[32 + bt]);
                  y[u] = ok ? silu_half(h) : 0.f;
                }
                pk[e / 2] = pack_bf16(y[0], y[1]);
              }
            }
            tmem_st4(pbuf + c8 * 4, pk);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&p_full[buf]);
          mbar_arrive(&ts_free[kst]);
        }
      }
      if (fail) break;
      n += nk;
      // ---- epilogue: this warpgroup's half of O = (1/N) (P V [+ self term])
      float* O = static_cast<float*>(a.o);
      const int h = item.h;
      float self_w = 0.f;
      if (cand && rvalid && row_in) {
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
        self_w = silu_acc(sdot + rab[0] + rab[32]);
      }
      if (nk > 0) {
        fail = !mbar_wait(o_full, items_done & 1, abort_flag, P.status);
        ++items_done;
        if (named_barrier_any(bid, 128, fail)) break;
        tc_fence_after();
      }
      const bf16* sv = static_cast<const bf16*>(a.self_v) + (g.qs + r0 + row) * a.q_stride + h * DH;
      const int odh = a.o_dh > 0 ? a.o_dh : DH;       // O columns stored per head
#pragma unroll
      for (int cc = 0; cc < DH / 64; ++cc) {
        const int c = wg * (DH / 64) + cc;            // 32-column chunk of O
        if (c * 32 >= odh) continue;                   // zero-padded head columns
        float o[32];
        if (nk > 0) {
          uint32_t r[32];
          tmem_ld32(tO + lane_off + c * 32, r);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __uint_as_float(r[i]);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0.f;
        }
        if (rvalid && row_in &&
            bounds_ok(h * odh + c * 32 + 32 <= a.o_stride && h * DH + c * 32 + 32 <= a.q_stride,
                      P.status)) {
          if (cand) {
#pragma unroll
            for (int i = 0; i < 32; i += 8) {
              const uint4 va = *reinterpret_cast<const uint4*>(sv + c * 32 + i);
              const __nv_bfloat162* vh = reinterpret_cast<const __nv_bfloat162*>(&va);
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                const float2 vf = __bfloat1622float2(vh[u]);
                o[i + 2 * u] = fmaf(self_w, vf.x, o[i + 2 * u]);
                o[i + 2 * u + 1] = fmaf(self_w, vf.y, o[i + 2 * u + 1]);
              }
            }
          }
          float* dst = O + (g.qs + r0 + row) * a.o_stride + h * odh + c * 32;
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(dst + i) =
                make_float4(o[i] * a.inv_N, o[i + 1] * a.inv_N, o[i + 2] * a.inv_N, o[i + 3] * a.inv_N);
        }
      }
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
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

int sm_count_attn() {
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
cudaError_t launch_fwd(const AttnArgs& a, void* ws, uint32_t* status, cudaStream_t s) {
  using C = FwdCfg<DH>;
  // Tensor maps over the Q block of the query rows' G and the K and V blocks
  // of the key rows: each starts at its block's head-0 column, d columns wide,
  // rows q_stride / kv_stride elements apart; a box is 64 columns x 128 rows.
  const int d = a.H * DH;
  CUtensorMap tQ, tK, tV;
  const bf16* q = static_cast<const bf16*>(a.q);
  const bf16* k = static_cast<const bf16*>(a.k);
  const bf16* v = static_cast<const bf16*>(a.v);
  FwdParams P;
  P.a = a;
  P.w = sched_ws(ws);
  P.status = status;
  bool ok = encode_tmap_2d(&tQ, false, q, (uint64_t)d, (uint64_t)a.q_rows, (uint64_t)a.q_stride, 64, kTile) &&
            encode_tmap_2d(&tK, false, k, (uint64_t)d, (uint64_t)a.kv_rows, (uint64_t)a.kv_stride, 64, kTile) &&
            encode_tmap_2d(&tV, false, v, (uint64_t)d, (uint64_t)a.kv_rows, (uint64_t)a.kv_stride, 64, kTile);
  if (!ok) return cudaErrorInvalidValue;
  cudaError_t e = build_schedule(a, ws, s);
  if (e != cudaSuccess) return e;
  auto kern = attn_fwd_tc_kernel<DH>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  kern<<<sm_count_attn(), C::THREADS, C::SMEM, s>>>(tQ, tK, tV, P);
  count_launch();
  return cudaGetLastError();
}

}  // namespace

bool attention_fwd_tc_supported(int dtype, const AttnArgs& a) {
  return dtype == HSTU_BF16 && (a.dh == 64 || a.dh == 128) && a.q_rows > 0 && a.kv_rows > 0 &&
         a.q_stride % 8 == 0 && a.kv_stride % 8 == 0 && a.P <= 32 && a.Bt <= 32;
}

cudaError_t attention_fwd_tc(const AttnArgs& a, void* ws, uint32_t* status, cudaStream_t s) {
  if (a.dh == 128) return launch_fwd<128>(a, ws, status, s);
  return launch_fwd<64>(a, ws, status, s);
}

}  // namespace hstu

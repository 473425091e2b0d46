// Tensor-core (tcgen05) GEMM with the projection epilogues of the HSTU layer.
//
//   C[M][N] = A(M x K) B(K x N), bf16 operands, fp32 accumulation in TMEM.
//
// Used for equation (1) of the HSTU walkthrough (X W1 with the SiLU and
// U|V|Q|K split fused into the epilogue), equation (3)'s output projection
// (Z W2 + b2 + X, residual fused), and the backward contractions (dY W2^T,
// dPre W1^T + dY, and the split-K weight gradients Z^T dY, X^T dPre reduced
// with TMA reduce-add into fp32).
//
// Persistent, warp-specialised CTA of 6 warps on one SM:
//   warp 0      TMA producer: 128x64 A and BNx64 B tiles into a ring of stages
//   warp 1      MMA issuer: 4 x tcgen05.mma (128 x BN x 16) per stage into a
//               double-buffered TMEM accumulator
//   warps 2..9  epilogue, two warpgroups taking alternate 128-byte-wide
//               chunks of each tile: tcgen05.ld of their 32 TMEM lanes, bias /
//               SiLU / residual, 128-byte-swizzled staging in shared memory
//               (one staging tile per warpgroup), TMA store (or TMA reduce-add
//               for split-K); a warpgroup waits for its previous store only
//               when it next needs its staging tile
// PAIR: a cluster of two CTAs computes 256-row tiles with tcgen05 cta_group::2:
// each CTA loads its own 128 rows of A and half of the tile's B columns, the
// even CTA's MMA thread issues M = 256 MMAs over both SMs' shared memory and
// TMEM (each CTA holds the accumulator rows of its A rows), its commits arrive
// on both CTAs' barriers, and both CTAs' loads and epilogues report to the
// even CTA's barriers.  Per SM this halves the B operand's shared-memory
// reads and the TMA traffic of B.  No load multicasts.
// Every mbarrier wait is bounded; a timeout sets the library's device status
// word and the CTA drains its own copies and MMAs, frees its TMEM and exits.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace hstu {
namespace {

using namespace tc;

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int kThreads = 320;
constexpr int kMaxSmem = 232448;

template <int BN, bool AK, bool BKM, int EPI, typename TOUT, bool PAIR>
struct Cfg {
  static constexpr int A_BYTES = BM * 128;
  static constexpr int B_BYTES = (PAIR ? BN / 2 : BN) * 128;   // this CTA's part of the B tile
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int NOUT = EPI == EPI_SILU_SPLIT ? 2 : 1;
  static constexpr int OUT_ES = (int)sizeof(TOUT);
  static constexpr int CW = 128 / OUT_ES;  // columns per staged chunk (128 bytes per row)
  static constexpr int STG_BYTES = BM * 128;
  static constexpr int BAR_BYTES = 1024;
  static constexpr int STAGES_FIT = (kMaxSmem - 1024 - 2 * NOUT * STG_BYTES - BAR_BYTES) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_FIT > 6 ? 6 : STAGES_FIT;
  static constexpr int SMEM = 1024 /*align slack*/ + STAGES * STAGE_BYTES + 2 * NOUT * STG_BYTES + BAR_BYTES;
  static constexpr uint32_t IDESC = idesc_bf16(PAIR ? 2 * BM : BM, BN, !AK, !BKM);
  static_assert(STAGES >= 2, "not enough shared memory for two stages");
  static_assert(BN % CW == 0 || CW > BN, "chunking");
};

struct KParams {
  int64_t M, N, K;
  int n_tiles;          // tiles along N
  int tiles;            // total output tiles
  int ksplit;           // K chunks per tile
  int kb_per_split;     // k-blocks per chunk
  int total_kb;         // k-blocks of the whole K
  const void* bias;     // [N] bf16 or null
  uint32_t* status;
  bool has_c;           // SILU_SPLIT: write Pre too
  void* c2;             // RESID with fp32 output: also a bf16 copy of C here (or null)
  int64_t ldc2;
};

// SiLU(x) = h + h tanh(h) with h = x / 2 (x sigmoid(x), as an identity).
__device__ __forceinline__ float silu_tanh(float x) {
  const float h = 0.5f * x;
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(h));
  return fmaf(h, t, h);
}

__device__ __forceinline__ float bf16_bits_to_f(uint16_t b) {
  return __uint_as_float(((uint32_t)b) << 16);
}

template <int BN, bool AK, bool BKM, int EPI, typename TOUT, bool PAIR>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmC2,
                   const __grid_constant__ CUtensorMap tmR, const KParams p) {
  using C = Cfg<BN, AK, BKM, EPI, TOUT, PAIR>;
  // Tiles need a 1024-byte aligned base; using the array itself (not an
  // address rounded through an integer) keeps the pointers below in the
  // shared state space, so staging accesses compile to shared, not generic,
  // instructions.
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {              // uniform over the block: all threads leave
    if (threadIdx.x == 0 && p.status) atomicOr(p.status, kStatusSmemAlign);
    return;
  }
  uint8_t* smem = smem_raw;
  uint8_t* stages = smem;
  uint8_t* stg = smem + C::STAGES * C::STAGE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(stg + 2 * C::NOUT * C::STG_BYTES);
  uint64_t* full = bars;                       // [STAGES]
  uint64_t* empty = bars + C::STAGES;          // [STAGES]
  uint64_t* acc_full = empty + C::STAGES;      // [2]
  uint64_t* acc_empty = acc_full + 2;          // [2]
  uint64_t* res_bar = acc_empty + 2;           // [2] one per epilogue warpgroup
  uint64_t* done_bar = res_bar + 2;            // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int units = p.tiles * p.ksplit;
  // PAIR: the two CTAs of a cluster walk the same units; rank picks the rows
  const uint32_t rank = PAIR ? cluster_rank() : 0u;
  const bool leader = rank == 0;
  const int u_first = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int u_step = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  constexpr int TM = PAIR ? 2 * BM : BM;               // rows per tile

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], PAIR ? 16 : 8);     // epilogue warps (of both CTAs)
    }
    mbar_init(&res_bar[0], 1);
    mbar_init(&res_bar[1], 1);
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    if (PAIR) tmem_alloc_pair(tmem_slot, 2 * BN);
    else tmem_alloc(tmem_slot, 2 * BN);
  }
  tc_fence_before();
  __syncthreads();
  if (PAIR) cluster_sync();                    // both CTAs' barriers exist before any remote use
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0;        // bit s: stage s holds a load that may be unconsumed
      uint32_t issued_par = 0;    // bit s: phase parity of that load
      for (int u = u_first; u < units && !*abort_flag; u += u_step) {
        const int tile = u % p.tiles, ks = u / p.tiles;
        const int m0 = (tile / p.n_tiles) * TM + (int)rank * BM, n0 = (tile % p.n_tiles) * BN;
        const int kb0 = ks * p.kb_per_split;
        const int kb1 = min(p.total_kb, kb0 + p.kb_per_split);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.status)) break;
          uint8_t* sA = stages + stage * C::STAGE_BYTES;
          uint8_t* sB = sA + C::A_BYTES;
          if (PAIR) {
            // both CTAs' bytes land on the even CTA's barrier
            const uint32_t cfull = cluster_addr(&full[stage], 0);
            if (leader) mbar_expect_tx(&full[stage], 2 * C::STAGE_BYTES);
            const int nb = n0 + (int)rank * (BN / 2);
            if (AK) {
              tma_load_2d_pair(sA, &tmA, cfull, kb * BK, m0);
            } else {
              tma_load_2d_pair(sA, &tmA, cfull, m0, kb * BK);
              tma_load_2d_pair(sA + 8192, &tmA, cfull, m0 + 64, kb * BK);
            }
            if (BKM) {
              tma_load_2d_pair(sB, &tmB, cfull, kb * BK, nb);
            } else {
#pragma unroll
              for (int j = 0; j < BN / 128; ++j)
                tma_load_2d_pair(sB + j * 8192, &tmB, cfull, nb + 64 * j, kb * BK);
            }
            issued |= 1u << stage;
            issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
            if (++stage == C::STAGES) {
              stage = 0;
              phase ^= 1;
            }
            continue;
          }
          mbar_expect_tx(&full[stage], C::STAGE_BYTES);
          if (AK) {
            tma_load_2d(sA, &tmA, &full[stage], kb * BK, m0);
          } else {
            tma_load_2d(sA, &tmA, &full[stage], m0, kb * BK);
            tma_load_2d(sA + 8192, &tmA, &full[stage], m0 + 64, kb * BK);
          }
          if (BKM) {
            tma_load_2d(sB, &tmB, &full[stage], kb * BK, n0);
          } else {
#pragma unroll
            for (int j = 0; j < BN / 64; ++j)
              tma_load_2d(sB + j * 8192, &tmB, &full[stage], n0 + 64 * j, kb * BK);
          }
          issued |= 1u << stage;
          issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // drain: every load this thread issued has landed before the CTA exits
      // (PAIR: the even CTA's barriers count both CTAs' loads)
      for (int s = 0; s < C::STAGES; ++s)
        if (leader && (issued & (1u << s))) {
          volatile int never = 0;
          mbar_wait(&full[s], (issued_par >> s) & 1u, &never, p.status);
        }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && leader) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      for (int u = u_first; u < units && !*abort_flag; u += u_step) {
        const int ks = u / p.tiles;
        const int kb0 = ks * p.kb_per_split;
        const int kb1 = min(p.total_kb, kb0 + p.kb_per_split);
        if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1, abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        bool ok = true;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(stages + stage * C::STAGE_BYTES);
          const uint32_t b0 = a0 + C::A_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t ad = AK ? sdesc_kmajor(a0 + k * 32) : sdesc_mnmajor(a0 + k * 2048, 8192);
            const uint64_t bd = BKM ? sdesc_kmajor(b0 + k * 32) : sdesc_mnmajor(b0 + k * 2048, 8192);
            if (PAIR) mma_ss_pair(d_tmem, ad, bd, C::IDESC, (kb > kb0 || k > 0) ? 1u : 0u);
            else mma_ss(d_tmem, ad, bd, C::IDESC, (kb > kb0 || k > 0) ? 1u : 0u);
          }
          if (PAIR) mma_commit_pair(&empty[stage], 0x3);
          else mma_commit(&empty[stage]);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        if (PAIR) mma_commit_pair(&acc_full[acc], 0x3);
        else mma_commit(&acc_full[acc]);
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1;
        }
      }
      // drain: all MMAs issued by this thread complete before TMEM is freed
      if (PAIR) mma_commit_pair(done_bar, 0x1);
      else mma_commit(done_bar);
      volatile int never = 0;
      mbar_wait(done_bar, 0, &never, p.status);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;             // chunks half, half + 2, ...
    const int row = quarter * 32 + lane;          // accumulator row (TMEM lane)
    const int et = (threadIdx.x - 64) & 127;      // thread in the warpgroup
    const uint32_t bid = 1 + half;                // this warpgroup's named barrier
    uint8_t* const wstg = stg + half * C::NOUT * C::STG_BYTES;
    uint64_t* const wres = res_bar + half;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    int acc = 0;
    uint32_t acc_phase = 0;
    uint32_t res_phase = 0;
    const uint32_t c_acc_empty0 = PAIR ? cluster_addr(&acc_empty[0], 0) : 0u;
    for (int u = u_first; u < units; u += u_step) {
      const int tile = u % p.tiles;
      const int m0 = (tile / p.n_tiles) * TM + (int)rank * BM, n0 = (tile % p.n_tiles) * BN;
      if (EPI == EPI_RESID && et == 0) {
        // this warpgroup's residual chunks of the tile into L2 before the accumulator is ready
        for (int c0 = half * C::CW; c0 < BN && c0 < p.N - n0; c0 += 2 * C::CW) tma_prefetch_2d(&tmR, n0 + c0, m0);
      }
      bool fail = *abort_flag != 0;
      if (!fail) fail = !mbar_wait(&acc_full[acc], acc_phase, abort_flag, p.status);
      if (named_barrier_any(bid, 128, fail)) break;
      tc_fence_after();
      const uint32_t t_acc = tmem_base + lane_off + acc * BN;
      bool ok = true;
#pragma unroll 1
      for (int c0 = half * C::CW; c0 < BN; c0 += 2 * C::CW) {
        if (c0 >= p.N - n0) break;   // chunk entirely past N
        float v[C::CW];
        {
          uint32_t r[32];
#pragma unroll
          for (int h = 0; h < C::CW / 32; ++h) {
            tmem_ld32(t_acc + c0 + 32 * h, r);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) v[32 * h + i] = __uint_as_float(r[i]);
          }
        }
        if (p.bias && EPI != EPI_ATOMIC_F32) {
          const uint16_t* b16 = static_cast<const uint16_t*>(p.bias);
#pragma unroll
          for (int i = 0; i < C::CW; ++i) {
            const int64_t n = n0 + c0 + i;
            v[i] += n < p.N ? bf16_bits_to_f(__ldg(b16 + n)) : 0.f;
          }
        }
        // the staging tile is free once this warpgroup's previous store has read it
        if (et == 0) bulk_wait_read0();
        named_barrier(bid, 128);
        if (EPI == EPI_RESID) {
          if (et == 0) {
            mbar_expect_tx(wres, C::STG_BYTES);
            tma_load_2d(wstg, &tmR, wres, n0 + c0, m0);
          }
          const bool fail_r = !mbar_wait(wres, res_phase, abort_flag, p.status);
          res_phase ^= 1;
          if (named_barrier_any(bid, 128, fail_r)) {
            ok = false;
            break;
          }
        }
        // write the staged chunk(s): row `row`, 16-byte pieces
        if (EPI == EPI_SILU_SPLIT) {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            uint4 pre, g;
            uint32_t* pp = reinterpret_cast<uint32_t*>(&pre);
            uint32_t* gg = reinterpret_cast<uint32_t*>(&g);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float x0 = v[8 * j + 2 * q], x1 = v[8 * j + 2 * q + 1];
              pp[q] = pack_bf16(x0, x1);
              gg[q] = pack_bf16(silu_tanh(x0), silu_tanh(x1));
            }
            *reinterpret_cast<uint4*>(wstg + sw128(row, j)) = g;
            *reinterpret_cast<uint4*>(wstg + C::STG_BYTES + sw128(row, j)) = pre;
          }
        } else if (C::OUT_ES == 2) {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            uint4 o;
            uint32_t* oo = reinterpret_cast<uint32_t*>(&o);
            if (EPI == EPI_RESID) {
              const uint4 rr = *reinterpret_cast<const uint4*>(wstg + sw128(row, j));
              const uint32_t* rw = reinterpret_cast<const uint32_t*>(&rr);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const float r0 = __uint_as_float(rw[q] << 16), r1 = __uint_as_float(rw[q] & 0xFFFF0000u);
                oo[q] = pack_bf16(v[8 * j + 2 * q] + r0, v[8 * j + 2 * q + 1] + r1);
              }
            } else {
#pragma unroll
              for (int q = 0; q < 4; ++q) oo[q] = pack_bf16(v[8 * j + 2 * q], v[8 * j + 2 * q + 1]);
            }
            *reinterpret_cast<uint4*>(wstg + sw128(row, j)) = o;
          }
        } else {
          uint32_t lo[16];   // RESID: the chunk's row rounded to bf16 for the copy in c2
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            float4 o = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
            if (EPI == EPI_RESID) {
              const float4 rr = *reinterpret_cast<const float4*>(wstg + sw128(row, j));
              o.x += rr.x; o.y += rr.y; o.z += rr.z; o.w += rr.w;
              lo[2 * j] = pack_bf16(o.x, o.y);
              lo[2 * j + 1] = pack_bf16(o.z, o.w);
            }
            *reinterpret_cast<float4*>(wstg + sw128(row, j)) = o;
          }
          if (EPI == EPI_RESID && p.c2 != nullptr && m0 + row < p.M) {
            // 16-byte pieces straight to global (N is a multiple of 16, so a
            // piece of 8 columns is wholly inside or outside the matrix)
            bf16* dst = static_cast<bf16*>(p.c2) + (int64_t)(m0 + row) * p.ldc2 + n0 + c0;
#pragma unroll
            for (int q = 0; q < 4; ++q)
              if (n0 + c0 + 8 * q < p.N)
                *reinterpret_cast<uint4*>(dst + 8 * q) =
                    make_uint4(lo[4 * q], lo[4 * q + 1], lo[4 * q + 2], lo[4 * q + 3]);
          }
        }
        fence_proxy_async_smem();
        named_barrier(bid, 128);
        if (et == 0) {
          if (EPI == EPI_ATOMIC_F32) {
            tma_reduce_add_2d(&tmC, wstg, n0 + c0, m0);
          } else if (EPI == EPI_SILU_SPLIT) {
            tma_store_2d(&tmC2, wstg, n0 + c0, m0);
            if (p.has_c) tma_store_2d(&tmC, wstg + C::STG_BYTES, n0 + c0, m0);
          } else {
            tma_store_2d(&tmC, wstg, n0 + c0, m0);
          }
          bulk_commit();
        }
      }
      if (!ok) break;
      // accumulator buffer free for the MMA warp
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (PAIR) mbar_arrive_cluster(c_acc_empty0 + (uint32_t)(acc * sizeof(uint64_t)));
        else mbar_arrive(&acc_empty[acc]);
      }
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
    if (et == 0) bulk_wait0();
  }

  tc_fence_before();
  __syncthreads();
  if (PAIR) cluster_sync();                    // no CTA leaves while its pair may still use it
  if (warp == 1) {
    tc_fence_after();
    if (PAIR) tmem_dealloc_pair(tmem_base, 2 * BN);
    else tmem_dealloc(tmem_base, 2 * BN);
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
int sm_count() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

template <int BN, bool AK, bool BKM, int EPI, typename TOUT, bool PAIR>
cudaError_t run_cfg(const GemmArgs& g, uint32_t* status, cudaStream_t s) {
  using Cf = Cfg<BN, AK, BKM, EPI, TOUT, PAIR>;
  CUtensorMap tA, tB, tC, tC2, tR;
  memset(&tC, 0, sizeof(tC));
  memset(&tC2, 0, sizeof(tC2));
  memset(&tR, 0, sizeof(tR));
  bool ok = AK ? encode_tmap_2d(&tA, false, g.A, g.K, g.M, g.lda, 64, BM)
               : encode_tmap_2d(&tA, false, g.A, g.M, g.K, g.lda, 64, 64);
  ok = ok && (BKM ? encode_tmap_2d(&tB, false, g.B, g.K, g.N, g.ldb, 64, PAIR ? BN / 2 : BN)
                  : encode_tmap_2d(&tB, false, g.B, g.N, g.K, g.ldb, 64, 64));
  const bool o32 = sizeof(TOUT) == 4;
  if (EPI == EPI_ATOMIC_F32) {
    ok = ok && encode_tmap_2d(&tC, true, g.Cf, g.N, g.M, g.ldc, Cf::CW, BM);
  } else if (EPI == EPI_SILU_SPLIT) {
    ok = ok && encode_tmap_2d(&tC2, false, g.C2, g.N, g.M, g.ldc, Cf::CW, BM);
    if (g.C) ok = ok && encode_tmap_2d(&tC, false, g.C, g.N, g.M, g.ldc, Cf::CW, BM);
  } else {
    ok = ok && encode_tmap_2d(&tC, o32, g.C, g.N, g.M, g.ldc, Cf::CW, BM);
    if (EPI == EPI_RESID) ok = ok && encode_tmap_2d(&tR, o32, g.R, g.N, g.M, g.ldr, Cf::CW, BM);
  }
  if (!ok) return cudaErrorInvalidValue;

  KParams p;
  p.M = g.M;
  p.N = g.N;
  p.K = g.K;
  p.n_tiles = (int)((g.N + BN - 1) / BN);
  constexpr int TMR = PAIR ? 2 * BM : BM;
  const int m_tiles = (int)((g.M + TMR - 1) / TMR);
  p.tiles = p.n_tiles * m_tiles;
  p.total_kb = (int)((g.K + BK - 1) / BK);
  p.ksplit = 1;
  if (EPI == EPI_ATOMIC_F32) {
    // enough (tile, K-chunk) units for two waves, chunks of at least 8 k-blocks
    const int want = 2 * sm_count();
    int ks = (want + p.tiles - 1) / p.tiles;
    const int maxks = p.total_kb / 8 > 0 ? p.total_kb / 8 : 1;
    p.ksplit = ks < 1 ? 1 : (ks > maxks ? maxks : ks);
  }
  p.kb_per_split = (p.total_kb + p.ksplit - 1) / p.ksplit;
  p.ksplit = (p.total_kb + p.kb_per_split - 1) / p.kb_per_split;  // no empty chunk
  p.bias = g.bias;
  p.status = status;
  p.has_c = g.C != nullptr;
  p.c2 = (EPI == EPI_RESID && o32) ? g.C2 : nullptr;
  p.ldc2 = g.ldc;
  const int units = p.tiles * p.ksplit;
  auto kern = gemm_tc_kernel<BN, AK, BKM, EPI, TOUT, PAIR>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cf::SMEM);
  if (e != cudaSuccess) return e;
  if (PAIR) {
    // clusters of two CTAs, one pair per two SMs
    int pairs = sm_count() / 2;
    if (units < pairs) pairs = units;
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3((unsigned)(2 * pairs));
    lc.blockDim = dim3(kThreads);
    lc.dynamicSmemBytes = Cf::SMEM;
    lc.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 2;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    lc.attrs = at;
    lc.numAttrs = 1;
    e = cudaLaunchKernelEx(&lc, kern, tA, tB, tC, tC2, tR, p);
    if (e != cudaSuccess) return e;
  } else {
    int grid = sm_count();
    if (units < grid) grid = units;
    kern<<<grid, kThreads, Cf::SMEM, s>>>(tA, tB, tC, tC2, tR, p);
  }
  count_launch();
  return cudaGetLastError();
}

// 256-wide tiles on CTA pairs once there are enough rows for them (a short-K
// residual GEMM, bound by its epilogue, stays on single CTAs)
template <int BN, bool AK, bool BKM, int EPI, typename TOUT>
cudaError_t run(const GemmArgs& g, uint32_t* status, cudaStream_t s) {
  const bool pair = BN == 256 && g.M >= 2 * BM && !(EPI == EPI_RESID && g.K < 2048);
  if (pair) return run_cfg<BN, AK, BKM, EPI, TOUT, true>(g, status, s);
  return run_cfg<BN, AK, BKM, EPI, TOUT, false>(g, status, s);
}

template <int BN>
cudaError_t dispatch_bn(const GemmArgs& g, uint32_t* st, cudaStream_t s) {
  const bool io32 = g.io_f32;
  if (g.epi == EPI_ATOMIC_F32) {
    if (!g.a_kmajor && !g.b_kmajor) return run<BN, false, false, EPI_ATOMIC_F32, float>(g, st, s);
    return cudaErrorNotSupported;
  }
  if (!g.a_kmajor) return cudaErrorNotSupported;
  if (g.epi == EPI_SILU_SPLIT) {
    if (!g.b_kmajor) return run<BN, true, false, EPI_SILU_SPLIT, bf16>(g, st, s);
    return cudaErrorNotSupported;
  }
  if (g.epi == EPI_RESID) {
    if (g.b_kmajor)
      return io32 ? run<BN, true, true, EPI_RESID, float>(g, st, s) : run<BN, true, true, EPI_RESID, bf16>(g, st, s);
    return io32 ? run<BN, true, false, EPI_RESID, float>(g, st, s) : run<BN, true, false, EPI_RESID, bf16>(g, st, s);
  }
  if (g.epi == EPI_STORE) {
    if (g.b_kmajor)
      return io32 ? run<BN, true, true, EPI_STORE, float>(g, st, s) : run<BN, true, true, EPI_STORE, bf16>(g, st, s);
    return io32 ? run<BN, true, false, EPI_STORE, float>(g, st, s) : run<BN, true, false, EPI_STORE, bf16>(g, st, s);
  }
  return cudaErrorNotSupported;
}

}  // namespace

// Shapes the tensor-core GEMM takes: bf16 operands, 16-byte-aligned rows,
// N a multiple of 16, no bias with split-K.
bool gemm_tc_supported(int dtype, const GemmArgs& g) {
  if (dtype != HSTU_BF16) return false;
  if (g.M <= 0 || g.N <= 0 || g.K <= 0) return false;
  if (g.N % 16 != 0 || g.lda % 8 != 0 || g.ldb % 8 != 0 || g.ldc % 8 != 0) return false;
  if (g.epi == EPI_RESID && g.ldr % 8 != 0) return false;
  if (g.epi == EPI_ATOMIC_F32) return !g.a_kmajor && !g.b_kmajor;
  if (!g.a_kmajor) return false;
  if (g.epi == EPI_SILU_SPLIT) return !g.b_kmajor;
  return true;
}

cudaError_t gemm_tc(const GemmArgs& g, uint32_t* status, cudaStream_t s) {
  if (g.N >= 256) return dispatch_bn<256>(g, status, s);
  if (g.N > 64) return dispatch_bn<128>(g, status, s);
  return dispatch_bn<64>(g, status, s);
}

}  // namespace hstu

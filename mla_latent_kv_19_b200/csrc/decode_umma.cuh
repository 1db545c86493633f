// Split-KV MLA decode over the paged latent cache on 5th-generation tensor
// cores (tcgen05 + TMEM + TMA), for the DeepSeek-V2 shape: H = 128 query
// heads, latent rows of D = d_c + d_r = 512 + 64 bf16 values, 64-token pages.
//
// Method (DeepSeek V2 MLA page, section 2.3): with W_UK absorbed into the
// query, every head scores s_hj = scale * q_lat_h . row_j over the shared
// latent rows, and with W_UV absorbed into the output the value of token j is
// row_j[0:512].  The 128 heads of one sequence form the M = 128 dimension of
// two dense contractions per 64-token page:  S = Q K^T (K = 576) and
// O += P V (N = 512).
//
// Why two CTAs per (sequence, split): the fp32 accumulator O (128 x 512) fills
// all 512 TMEM columns of an SM, and Q (128 x 576 bf16 = 144 KB) plus a 72 KB
// page does not leave room for a pipeline in one SM's shared memory.  A
// cluster of two CTAs splits the roles:
//
//   CTA 0 ("score"):  Q lives in TMEM (columns 0..287, two bf16 per column)
//     and is the A operand of TS-form UMMAs; pages stream through a 3-stage
//     TMA ring; S = Q K^T goes to one of two TMEM buffers (columns 384/448);
//     four softmax warps (one TMEM lane quadrant each, one head per thread)
//     run the online softmax and store P (bf16, UMMA K-major 128B-swizzled
//     layout) straight into CTA 1's shared memory.
//   CTA 1 ("value"):  O accumulates in TMEM columns 0..511; the same pages'
//     first 512 columns stream through a 2-stage TMA ring (an L2 hit after
//     CTA 0's read); P V is issued as two N = 256 SS-form UMMAs per 16-token
//     K step, V being the MN-major B operand.
//
// The running maximum is only moved when a tile's maximum exceeds it by more
// than 8 (log2 units), so P stays <= 256 and O needs rescaling (a TMEM read-
// modify-write by CTA 1's correction warps) only on those rare tiles; the
// final normalisation by the same running maximum makes the result exact.
//
// Every mbarrier wait is bounded (iterations and time): a wait that gives up
// records MLA_ERR_TIMEOUT, the roles stop, copies and MMAs in flight are
// drained, TMEM is released and the kernel returns.
#pragma once

#include "device_common.cuh"
#include "sm100_ptx.cuh"

namespace mla {
namespace dec {

constexpr int kH = 128, kDc = 512, kD = 576, kTok = 64;
constexpr int kBoxBytes = 64 * 128;                    // 64 rows x 64 bf16
constexpr int kKBoxes = 9, kVBoxes = 8;
constexpr int kKStageBytes = kKBoxes * kBoxBytes;      // 73728
constexpr int kVStageBytes = kVBoxes * kBoxBytes;      // 65536
constexpr int kKStages = 3, kVStages = 2;
constexpr int kPBytes = kH * kTok * 2;                 // 16384

// shared-memory map, offsets from a 1024-byte aligned base
constexpr int kOffK = 0;                               // CTA 0: K ring
constexpr int kOffV = 0;                               // CTA 1: V ring
constexpr int kOffP = kVStages * kVStageBytes;         // CTA 1: P[2]
constexpr int kOffAlpha = kOffP + 2 * kPBytes;         // CTA 1: alpha[2][128]
constexpr int kOffFlag = kOffAlpha + 2 * kH * 4;       // CTA 1: flag[2][4]
constexpr int kOffLfin = kOffFlag + 2 * 4 * 4;         // CTA 1: l[128]
constexpr int kRegionEnd = kKStages * kKStageBytes;    // 221184
static_assert(kOffLfin + kH * 4 <= kRegionEnd, "CTA 1 buffers overlap the barriers");

enum Bar {
  kKFull = 0, kKEmpty = 3, kSFull = 6, kSEmpty = 8, kPEmpty = 10, kQReady = 12,  // CTA 0
  kVFull = 13, kVEmpty = 15, kPFull = 17, kPVDone = 19, kCorrReq = 21,           // CTA 1
  kCorrDone = 22, kOFull = 23, kFin = 24,
  kDrain = 25, kNumBars = 26
};
constexpr int kOffBar = kRegionEnd;
constexpr int kOffMisc = kOffBar + kNumBars * 8;       // [0] tmem base, [1] abort, [2] corr tile
constexpr int kSmemBytes = kOffMisc + 64 + 1024;       // + slack for the 1024-byte alignment

// TMEM columns
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColQ = 0;                          // CTA 0: Q, 288 columns
constexpr uint32_t kColS = 384;                        // CTA 0: S[2], 64 columns each
constexpr uint32_t kColO = 0;                          // CTA 1: O, 512 columns

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;              // log2 units
constexpr uint64_t kWaitNs = 1000000000ull;            // 1 s per wait
constexpr uint32_t kDrainIters = 0xffffffffu;

struct Split {
  int b, split, len, p0, ntiles;
};

__device__ __forceinline__ Split split_of(const DecodeArgs& a, int pair, int* err_once) {
  Split s;
  s.b = pair / a.num_splits;
  s.split = pair % a.num_splits;
  int len = a.seq_lens[s.b];
  const int cap = a.max_blocks * kTok;
  if (len < 0 || len > cap) {
    *err_once = 1;
    len = len < 0 ? 0 : cap;
  }
  s.len = len;
  const int pages = (len + kTok - 1) / kTok;
  const int pps = (pages + a.num_splits - 1) / a.num_splits;
  s.p0 = s.split * pps;
  const int p1 = min(pages, s.p0 + pps);
  s.ntiles = max(0, p1 - s.p0);
  return s;
}

// Physical page of tile t and its number of valid tokens (0 for an invalid page,
// which is then read from page 0 and masked entirely).
__device__ __forceinline__ int tile_page(const DecodeArgs& a, const Split& s, int t, int* valid) {
  const int idx = s.p0 + t;
  const int pg = a.block_table[static_cast<long>(s.b) * a.max_blocks + idx];
  if (pg < 0 || pg >= a.num_blocks) {
    *valid = 0;
    return -1;
  }
  *valid = min(kTok, s.len - idx * kTok);
  return pg;
}

__global__ void __launch_bounds__(256, 1) __cluster_dims__(2, 1, 1)
    decode_umma_kernel(const __grid_constant__ CUtensorMap tmap, const DecodeArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sb = ptx::smem_u32(smem);
  const uint32_t rank = ptx::cluster_rank();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile uint32_t* misc = reinterpret_cast<volatile uint32_t*>(smem + kOffMisc);
  auto bar = [&](int i) -> uint32_t { return sb + kOffBar + 8u * static_cast<uint32_t>(i); };
  const uint32_t iters = a.wait_limit;

  int bad_len = 0;
  const Split sp = split_of(a, static_cast<int>(blockIdx.x >> 1), &bad_len);
  if (bad_len && threadIdx.x == 0 && rank == 0) report_error(a.err, MLA_ERR_BAD_INDEX);

  // bounded waits; a warp-uniform verdict, and the abort flag on failure
  auto fail = [&]() {
    misc[1] = 1u;
    report_error(a.err, MLA_ERR_TIMEOUT);
  };
  auto wait_local = [&](uint32_t b_, uint32_t par) -> bool {
    if (misc[1]) return false;
    const bool ok = ptx::mbar_wait<false>(b_, par, iters, kWaitNs);
    if (!ok) fail();
    return ok;
  };
  auto wait_remote = [&](uint32_t b_, uint32_t par) -> bool {
    if (misc[1]) return false;
    const bool ok = ptx::mbar_wait<true>(b_, par, iters, kWaitNs);
    if (!ok) fail();
    return ok;
  };
  auto drain = [&](uint32_t b_, uint32_t par) { ptx::mbar_wait<false>(b_, par, kDrainIters, kWaitNs); };

  if (threadIdx.x == 0) {
    // CTA 0
    for (int i = 0; i < kKStages; ++i) {
      ptx::mbar_init(bar(kKFull + i), 1);
      ptx::mbar_init(bar(kKEmpty + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(bar(kSFull + i), 1);
      ptx::mbar_init(bar(kSEmpty + i), 128);
      ptx::mbar_init(bar(kPEmpty + i), 1);
    }
    ptx::mbar_init(bar(kQReady), 128);
    // CTA 1
    for (int i = 0; i < kVStages; ++i) {
      ptx::mbar_init(bar(kVFull + i), 1);
      ptx::mbar_init(bar(kVEmpty + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(bar(kPFull + i), 128);
      ptx::mbar_init(bar(kPVDone + i), 1);
    }
    ptx::mbar_init(bar(kCorrReq), 1);
    ptx::mbar_init(bar(kCorrDone), 128);
    ptx::mbar_init(bar(kOFull), 1);
    ptx::mbar_init(bar(kFin), 128);
    ptx::mbar_init(bar(kDrain), 1);
    misc[1] = 0u;
    misc[2] = 0u;
    ptx::fence_mbar_init_cluster();
  }
  if (warp == 1) {
    ptx::tmem_alloc(sb + kOffMisc, kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();       // the peer's barriers exist before any remote arrive
  ptx::tc_fence_after();
  const uint32_t tmem = misc[0];

  if (rank == 0) {
    // =========================== CTA 0: scores and softmax ===========================
    if (warp == 0 && lane == 0) {
      // TMA producer: full 576-column pages
      ptx::prefetch_tmap(&tmap);
      int issued = 0;
      for (int t = 0; t < sp.ntiles; ++t) {
        const int st = t % kKStages;
        if (!wait_local(bar(kKEmpty + st), ((t / kKStages) & 1) ^ 1)) break;
        int valid;
        int pg = tile_page(a, sp, t, &valid);
        if (pg < 0) {
          report_error(a.err, MLA_ERR_BAD_INDEX);
          pg = 0;
        }
        ptx::mbar_arrive_expect_tx(bar(kKFull + st), kKStageBytes);
        const uint32_t dst = sb + kOffK + st * kKStageBytes;
        for (int i = 0; i < kKBoxes; ++i)
          ptx::tma_load_2d(dst + i * kBoxBytes, &tmap, bar(kKFull + st), i * 64, pg * kTok);
        issued = t + 1;
      }
      for (int t = max(0, issued - kKStages); t < issued; ++t)
        drain(bar(kKFull + t % kKStages), (t / kKStages) & 1);
    } else if (warp == 1) {
      // MMA issuer: S[i] = Q K^T, A = Q from TMEM, B = page from shared memory
      if (lane == 0) {
        constexpr uint32_t idS = ptx::idesc_bf16_f32(128, 64, false, false);
        if (wait_local(bar(kQReady), 0)) {
          for (int t = 0; t < sp.ntiles; ++t) {
            const int st = t % kKStages, i = t & 1;
            if (!wait_local(bar(kKFull + st), (t / kKStages) & 1)) break;
            if (!wait_local(bar(kSEmpty + i), ((t >> 1) & 1) ^ 1)) break;
            ptx::tc_fence_after();
            const uint32_t d = tmem + kColS + 64u * i;
            const uint32_t kb = sb + kOffK + st * kKStageBytes;
#pragma unroll 4
            for (int j = 0; j < kD / 16; ++j) {
              const uint64_t bd = ptx::sdesc_sw128(kb + (j >> 2) * kBoxBytes + (j & 3) * 32, 16, 1024);
              ptx::umma_ts(d, tmem + kColQ + 8u * j, bd, idS, j > 0 ? 1u : 0u);
            }
            ptx::umma_commit(bar(kSFull + i));
            ptx::umma_commit(bar(kKEmpty + st));
          }
        }
        ptx::umma_commit(bar(kDrain));
        drain(bar(kDrain), 0);
      }
      __syncwarp();
    } else if (warp >= 4) {
      // softmax warpgroup: thread = head row r, TMEM lane quadrant q
      const int q = warp & 3;
      const int r = q * 32 + lane;
      const uint32_t lb = static_cast<uint32_t>(q * 32) << 16;
      // Q (this sequence's 128 x 576 absorbed queries) -> TMEM, two bf16 per column
      {
        const uint4* qrow = reinterpret_cast<const uint4*>(
            reinterpret_cast<const __nv_bfloat16*>(a.q_lat) + (static_cast<long>(sp.b) * kH + r) * kD);
#pragma unroll 1
        for (int c = 0; c < kD / 64; ++c) {
          uint32_t v[32];
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint4 u = __ldg(qrow + c * 8 + k);
            v[4 * k] = u.x;
            v[4 * k + 1] = u.y;
            v[4 * k + 2] = u.z;
            v[4 * k + 3] = u.w;
          }
          ptx::tmem_st32(tmem + lb + kColQ + 32u * c, v);
        }
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        ptx::mbar_arrive(bar(kQReady));
      }
      const uint32_t rP = ptx::mapa(sb + kOffP, 1);
      const uint32_t rAlpha = ptx::mapa(sb + kOffAlpha, 1);
      const uint32_t rFlag = ptx::mapa(sb + kOffFlag, 1);
      const uint32_t rL = ptx::mapa(sb + kOffLfin, 1);
      const uint32_t rPFull = ptx::mapa(bar(kPFull), 1);
      const uint32_t rFin = ptx::mapa(bar(kFin), 1);
      const float sl2 = a.scale * kLog2e;
      float m_used = -INFINITY, l = 0.f;
#pragma unroll 1
      for (int t = 0; t < sp.ntiles; ++t) {
        const int i = t & 1;
        bool ok = wait_local(bar(kSFull + i), (t >> 1) & 1);
        if (!__all_sync(0xffffffffu, ok)) break;
        ptx::tc_fence_after();
        uint32_t s0[32], s1[32];
        ptx::tmem_ld32(tmem + lb + kColS + 64u * i, s0);
        ptx::tmem_ld32(tmem + lb + kColS + 64u * i + 32u, s1);
        ptx::tmem_wait_ld();
        ptx::tc_fence_before();
        ptx::mbar_arrive(bar(kSEmpty + i));
        int valid;
        tile_page(a, sp, t, &valid);
        float x[64];
        float m_tile = -INFINITY;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          x[j] = j < valid ? __uint_as_float(s0[j]) * sl2 : -INFINITY;
          x[j + 32] = j + 32 < valid ? __uint_as_float(s1[j]) * sl2 : -INFINITY;
          m_tile = fmaxf(m_tile, fmaxf(x[j], x[j + 32]));
        }
        const bool resc = m_tile > m_used + kRescaleThreshold;
        float alpha = 1.f;
        if (resc) {
          alpha = (m_used == -INFINITY) ? 0.f : exp2f(m_used - m_tile);
          m_used = m_tile;
        }
        uint32_t pk[32];
        float psum = 0.f;
        const bool live = m_used != -INFINITY;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float p0 = live ? exp2f(x[2 * j] - m_used) : 0.f;
          const float p1 = live ? exp2f(x[2 * j + 1] - m_used) : 0.f;
          const __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
          psum += __low2float(pb) + __high2float(pb);
          pk[j] = *reinterpret_cast<const uint32_t*>(&pb);
        }
        l = l * alpha + psum;
        ok = wait_remote(bar(kPEmpty + i), ((t >> 1) & 1) ^ 1);
        if (!__all_sync(0xffffffffu, ok)) break;
        // P row r into CTA 1: 8 chunks of 16 bytes, chunk index xor (row mod 8)
        const uint32_t prow = rP + i * kPBytes + r * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          ptx::st_cluster_v4(prow + ((c ^ (r & 7)) << 4), pk[4 * c], pk[4 * c + 1], pk[4 * c + 2],
                             pk[4 * c + 3]);
        ptx::st_cluster_u32(rAlpha + (i * kH + r) * 4, __float_as_uint(alpha));
        const unsigned any = __any_sync(0xffffffffu, resc && t > 0);
        if (lane == 0) ptx::st_cluster_u32(rFlag + (i * 4 + q) * 4, any);
        ptx::fence_proxy_async_cluster();
        ptx::mbar_arrive_remote(rPFull + 8u * i);
      }
      // this split's log-sum-exp (natural log) and the normaliser for CTA 1
      const long row = (static_cast<long>(sp.b) * a.num_splits + sp.split) * kH + r;
      a.lse_part[row] = l > 0.f ? (m_used + log2f(l)) * kLn2 : -INFINITY;
      ptx::st_cluster_u32(rL + r * 4, __float_as_uint(l));
      ptx::mbar_arrive_remote(rFin);
    }
  } else {
    // =========================== CTA 1: values ===========================
    if (warp == 0 && lane == 0) {
      // TMA producer: first 512 columns of the same pages
      ptx::prefetch_tmap(&tmap);
      int issued = 0;
      for (int t = 0; t < sp.ntiles; ++t) {
        const int st = t % kVStages;
        if (!wait_local(bar(kVEmpty + st), ((t / kVStages) & 1) ^ 1)) break;
        int valid;
        int pg = tile_page(a, sp, t, &valid);
        if (pg < 0) pg = 0;
        ptx::mbar_arrive_expect_tx(bar(kVFull + st), kVStageBytes);
        const uint32_t dst = sb + kOffV + st * kVStageBytes;
        for (int i = 0; i < kVBoxes; ++i)
          ptx::tma_load_2d(dst + i * kBoxBytes, &tmap, bar(kVFull + st), i * 64, pg * kTok);
        issued = t + 1;
      }
      for (int t = max(0, issued - kVStages); t < issued; ++t)
        drain(bar(kVFull + t % kVStages), (t / kVStages) & 1);
    } else if (warp == 1) {
      // MMA issuer: O += P V  (A = P, K-major; B = V, MN-major; two N = 256 halves)
      constexpr uint32_t idPV = ptx::idesc_bf16_f32(128, 256, false, true);
      int ncorr = 0;
#pragma unroll 1
      for (int t = 0; t < sp.ntiles; ++t) {
        const int st = t & 1;
        bool ok = wait_local(bar(kVFull + st), (t >> 1) & 1);
        ok = ok && wait_remote(bar(kPFull + st), (t >> 1) & 1);
        if (!__all_sync(0xffffffffu, ok)) break;
        int valid;
        tile_page(a, sp, t, &valid);
        if (valid < kTok) {
          // rows past the sequence end: zero them so that P = 0 meets finite V
          uint8_t* vs = smem + kOffV + st * kVStageBytes;
          const int n = (kTok - valid) * kVBoxes * 8;
          for (int idx = lane; idx < n; idx += 32) {
            const int chunk = idx & 7, box = (idx >> 3) & 7, rrow = valid + (idx >> 6);
            *reinterpret_cast<uint4*>(vs + box * kBoxBytes + rrow * 128 + chunk * 16) =
                make_uint4(0, 0, 0, 0);
          }
          ptx::fence_proxy_async_cta();
          __syncwarp();
        }
        const volatile uint32_t* fl = reinterpret_cast<const volatile uint32_t*>(smem + kOffFlag) + st * 4;
        const uint32_t flag = fl[0] | fl[1] | fl[2] | fl[3];
        if (flag) {
          if (lane == 0) {
            misc[2] = static_cast<uint32_t>(t);
            ptx::mbar_arrive(bar(kCorrReq));
          }
          ok = wait_local(bar(kCorrDone), ncorr & 1);
          ++ncorr;
          if (!__all_sync(0xffffffffu, ok)) break;
        }
        ptx::tc_fence_after();
        if (lane == 0) {
          ptx::fence_proxy_async_cta();
          const uint32_t pb = sb + kOffP + st * kPBytes;
          const uint32_t vb = sb + kOffV + st * kVStageBytes;
#pragma unroll
          for (int j = 0; j < kTok / 16; ++j) {
            const uint64_t ad = ptx::sdesc_sw128(pb + 32 * j, 16, 1024);
#pragma unroll
            for (int nh = 0; nh < 2; ++nh) {
              const uint64_t bd = ptx::sdesc_sw128(vb + nh * 4 * kBoxBytes + j * 2048, kBoxBytes, 1024);
              ptx::umma_ss(tmem + kColO + 256u * nh, ad, bd, idPV, (t > 0 || j > 0) ? 1u : 0u);
            }
          }
          ptx::umma_commit(bar(kPVDone + st));
        }
        __syncwarp();
      }
      if (lane == 0) {
        misc[2] = 0xffffffffu;            // no more correction requests
        ptx::mbar_arrive(bar(kCorrReq));
        ptx::umma_commit(bar(kOFull));
        ptx::umma_commit(bar(kDrain));    // TMEM stays allocated until every MMA is done
        drain(bar(kDrain), 0);
      }
      __syncwarp();
    } else if (warp == 2 && lane == 0) {
      // release: a finished P V frees its V stage here and its P buffer's producer in CTA 0
      const uint32_t rPEmpty = ptx::mapa(bar(kPEmpty), 0);
      for (int t = 0; t < sp.ntiles; ++t) {
        const int i = t & 1;
        if (!wait_local(bar(kPVDone + i), (t >> 1) & 1)) break;
        ptx::mbar_arrive(bar(kVEmpty + i));
        ptx::mbar_arrive_remote(rPEmpty + 8u * i);
      }
    } else if (warp >= 4) {
      // correction (rescale O rows on request) and epilogue
      const int q = warp & 3;
      const int r = q * 32 + lane;
      const uint32_t lb = static_cast<uint32_t>(q * 32) << 16;
      const float* alphas = reinterpret_cast<const float*>(smem + kOffAlpha);
      int k = 0;
#pragma unroll 1
      while (true) {
        bool ok = wait_local(bar(kCorrReq), k & 1);
        ++k;
        if (!__all_sync(0xffffffffu, ok)) break;
        const int t = static_cast<int>(misc[2]);
        if (t < 0) break;
        if (t >= 1) {
          ok = wait_local(bar(kPVDone + ((t - 1) & 1)), ((t - 1) >> 1) & 1);
          if (!__all_sync(0xffffffffu, ok)) break;
        }
        ptx::tc_fence_after();
        const float al = alphas[(t & 1) * kH + r];
#pragma unroll 1
        for (int c = 0; c < 16; ++c) {
          uint32_t v[32];
          ptx::tmem_ld32(tmem + lb + kColO + 32u * c, v);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * al);
          ptx::tmem_st32(tmem + lb + kColO + 32u * c, v);
        }
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        ptx::mbar_arrive(bar(kCorrDone));
      }
      bool ok = wait_local(bar(kOFull), 0);
      ok = ok && wait_remote(bar(kFin), 0);
      ok = __all_sync(0xffffffffu, ok);
      float* orow = a.o_part + ((static_cast<long>(sp.b) * a.num_splits + sp.split) * kH + r) * kDc;
      if (ok) {
        ptx::tc_fence_after();
        const float lsum = reinterpret_cast<const volatile float*>(smem + kOffLfin)[r];
        const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
        if (sp.ntiles == 0) {
          for (int c = 0; c < kDc; c += 4)
            *reinterpret_cast<float4*>(orow + c) = make_float4(0.f, 0.f, 0.f, 0.f);
        } else {
#pragma unroll 1
          for (int c = 0; c < 16; ++c) {
            uint32_t v[32];
            ptx::tmem_ld32(tmem + lb + kColO + 32u * c, v);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; e += 4)
              *reinterpret_cast<float4*>(orow + 32 * c + e) =
                  make_float4(__uint_as_float(v[e]) * inv, __uint_as_float(v[e + 1]) * inv,
                              __uint_as_float(v[e + 2]) * inv, __uint_as_float(v[e + 3]) * inv);
          }
        }
        ptx::tc_fence_before();
      }
    }
  }

  __syncthreads();
  ptx::cluster_sync();       // no remote access to this CTA's shared memory after this point
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace dec
}  // namespace mla

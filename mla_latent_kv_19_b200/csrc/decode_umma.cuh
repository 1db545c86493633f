// Split-KV MLA decode over the paged latent cache on 5th-generation tensor
// cores (tcgen05 + TMEM + TMA), for the DeepSeek-V2 shape: H = 128 query
// heads, latent rows of D = d_c + d_r = 512 + 64 values, 64-token pages.
//
// Method (DeepSeek V2 MLA page, section 2.3): with W_UK absorbed into the
// query, every head scores s_hj = scale * q_lat_h . row_j over the shared
// latent rows, and with W_UV absorbed into the output the value of token j is
// row_j[0:512].  The 128 heads of one sequence form the M = 128 dimension of
// two dense contractions per 64-token page:  S = Q K^T (K = 576) and
// O += P V (N = 512).
//
// Why two CTAs per (sequence, split): the fp32 accumulator O (128 x 512) fills
// all 512 TMEM columns of an SM, and Q (128 x 576 x 2 bytes = 144 KB) plus a
// 72 KB page does not leave room for a pipeline in one SM's shared memory.  A
// cluster of two CTAs splits the roles:
//
//   CTA 0 ("score"):  a ring of 3 shared-memory slots of 72 KB, each filled
//     by ONE 3-D TMA request that lands a whole page (64 rows x 576 columns)
//     as 9 column chunks of [64 rows x 128 bytes] with the 128-byte swizzle
//     (the UMMA K-major layout); the first two slots carry Q (two halves of
//     64 heads) into TMEM (columns 0..287, two values per column; Q is then
//     the A operand of TS-form UMMAs).  Two MMA warps, for even and odd tiles,
//     compute S = Q K^T (N = 64, one page per MMA) into two TMEM buffers
//     (columns 384/448); the commit that reports S also frees the page's slot.
//     Four softmax warps (one TMEM lane quadrant each, one head per thread) run
//     the online softmax and send their row of P (UMMA K-major swizzled
//     layout), the rescale factor and the warp's rescale flag to one of three
//     P buffers in CTA 1 with asynchronous distributed-shared-memory stores
//     (st.async), whose bytes CTA 1's barrier counts -- once P V has finished
//     reading that buffer's previous tile.  A slot is thus held only from its
//     load to the end of its MMAs.
//   CTA 1 ("value"):  O accumulates in TMEM columns 0..511; the same pages'
//     first 512 columns stream through a 2-stage ring, one 64 KB TMA request
//     per page (an L2 hit after CTA 0's read); P V is issued as two N = 256
//     SS-form UMMAs per 16-token K step, V being the MN-major B operand.
//
// e4m3 cache (kFp8): a page is 36,864 code bytes, fetched by one bulk copy
// into the upper half of its slot / the upper part of its stage; four
// converter warps per CTA expand the codes in place to fp16 (exact: an e4m3
// value has 4 significant bits and its exponent range lies inside fp16's) in
// the same swizzled layouts, with integer and fp16 arithmetic only.  The
// contractions then run with fp16 operands (Q is converted once, P is packed
// as fp16), and the per-token scale enters the softmax: the score of token j
// is scale_j times the score against its codes, and the P V operand carries
// p_j * scale_j while the normaliser sums p_j.
//
// Measured on B200: issuing a TMA request costs the producer a few hundred
// cycles (so requests are whole pages); a tcgen05.mma with M = 128 costs one
// issuing thread ~60 cycles whatever its N up to 128, while two threads issuing
// independent MMAs get through them twice as fast (hence N = 64 per page and
// two S issuers); a signal between the two CTAs of the cluster takes ~0.6 us
// (hence no round trip on a slot's way back to the producer); and the
// conversion / transcendental pipe is narrow (so the e4m3 codes are expanded
// with bit operations, leaving that pipe to the softmax's exponentials).
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

#include <cuda_fp16.h>

#include "device_common.cuh"
#include "sm100_ptx.cuh"

namespace mla {
namespace dec {

constexpr int kH = 128, kDc = 512, kD = 576, kTok = 64;
constexpr int kBoxBytes = 64 * 128;                    // 64 rows x 64 two-byte values (one column chunk)
constexpr int kKBoxes = 9, kVBoxes = 8;                // column chunks of a row / of V
constexpr int kSlotBytes = kKBoxes * kBoxBytes;        // 73728: 9 chunks x 64 rows x 128 B
constexpr int kChunkInSlot = kBoxBytes;                // 8192
constexpr int kQLoads = 2;                             // two halves of 64 heads
constexpr int kSlots = 3;                              // CTA 0 ring
constexpr int kVStageBytes = kVBoxes * kBoxBytes;      // 65536
constexpr int kVStages = 2;
constexpr int kPBytes = kH * kTok * 2;                 // 16384
constexpr int kPMsgBytes = kPBytes + kH * 4 + 16;      // P + alpha[128] + flag[4] = 16912
constexpr int kPBufStride = 17 * 1024;                 // keeps every P tile 1024-byte aligned
constexpr int kMaxTablePages = 512;                    // pages of a split kept in shared memory
// e4m3 cache: a page is 64 rows x 576 code bytes, contiguous in the pool, plus
// 64 fp32 per-token scales
constexpr int kPageF8Bytes = kTok * kD;                // 36864
constexpr int kF8InSlot = kSlotBytes - kPageF8Bytes;   // codes land in a slot's upper half
constexpr int kF8InStage = kVStageBytes - kPageF8Bytes;
constexpr int kScaleBytes = kTok * 4;
constexpr int kScaleRing = 6;                          // tile t's scales live in entry t % 6
constexpr int kF8UnitsK = kPageF8Bytes / 8 / 128;      // 36 eight-code units per converter thread
constexpr int kF8UnitsV = kTok * kDc / 8 / 128;        // 32 (V: first 512 columns)

// CTA 0 map
constexpr int kOffRing = 0;
constexpr int kOffTable0 = kSlots * kSlotBytes;        // 221184
// CTA 1 map
constexpr int kOffV = 0;
constexpr int kPBufs = 3;                              // tile t's P lives in buffer t % 3
constexpr int kOffP = kVStages * kVStageBytes;         // 131072: P buffers [3]
constexpr int kOffLfin = kOffP + kPBufs * kPBufStride; // l[128]
constexpr int kOffTable1 = kOffLfin + kH * 4;
constexpr int kRegionEnd = kOffTable0 + kMaxTablePages * 4;
static_assert(kOffTable1 + kMaxTablePages * 4 <= kRegionEnd, "CTA 1 map overlaps the barriers");

enum Bar {
  kFull = 0, kEmpty = kFull + kSlots,                                     // CTA 0 ring
  kSFull = kEmpty + kSlots, kSEmpty = kSFull + 2,                        // CTA 0
  kQReady = kSEmpty + 2,
  kPBufFree = kQReady + 1,                                                // CTA 0: CTA 1's P buffers
  kScl = kPBufFree + kPBufs,                                              // CTA 0: e4m3 scales ready
  kCvtLd = kScl + kScaleRing, kCvtDone = kCvtLd + 1,                     // e4m3 converters
  kVFull = kCvtDone + kSlots, kVEmpty = kVFull + kVStages,               // CTA 1
  kVCvt = kVEmpty + kVStages,
  kPFull = kVCvt + kVStages, kPVDone = kPFull + kPBufs,
  kCorrReq = kPVDone + 2, kCorrDone = kCorrReq + 1, kOFull = kCorrDone + 1, kFin = kOFull + 1,
  kDrain = kFin + 1, kDrain2 = kDrain + 1,                               // MMA issuers' drains
  kStgFull = kDrain2 + 1, kStgFree = kStgFull + 2,                       // CTA 0: bf16 P staging in TMEM
  kNumBars = kStgFree + 2
};
constexpr int kOffScale = kRegionEnd;                  // CTA 0: per-token scales [6][64]
constexpr int kOffStg = kOffScale + kScaleRing * kScaleBytes;  // CTA 0: staged alpha [2][128], flags [2][4]
constexpr int kOffBar = kOffStg + (2 * kH + 8) * 4;
// misc words: [0] tmem base, [1] abort, [2] corr tile, [3] P messages CTA 0 sent
// (written by CTA 0 into CTA 1), [4] messages CTA 1 consumed, [5] messages it armed
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmemBytes = kOffMisc + 64 + 1024;       // + slack for the 1024-byte alignment
static_assert(kSmemBytes <= 232448, "shared memory budget");

// TMEM columns
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColQ = 0;                          // CTA 0: Q, 288 columns
constexpr uint32_t kColS = 384;                        // CTA 0: S[2], 64 columns each
constexpr uint32_t kColStg = 288;                      // CTA 0 (bf16): staged P[2], 32 columns each
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

// Physical page of tile t (-1 if the table entry is outside the pool).
__device__ __forceinline__ int load_page(const DecodeArgs& a, const Split& s, int t) {
  const int pg = a.block_table[static_cast<long>(s.b) * a.max_blocks + s.p0 + t];
  return (pg < 0 || pg >= a.num_blocks) ? -1 : pg;
}

__device__ __forceinline__ int page_at(const DecodeArgs& a, const Split& s, const int* table, int t) {
  return t < kMaxTablePages ? table[t] : load_page(a, s, t);
}

__device__ __forceinline__ int valid_tokens(const Split& s, int page, int t) {
  return page < 0 ? 0 : min(kTok, s.len - (s.p0 + t) * kTok);
}

// Eight e4m3 codes (low byte first) to eight fp16 values with bit operations
// and one fp16 multiply per pair.  The fp16 bits (c & 0x7f) << 7 | (c & 0x80) << 8
// hold exactly value(c) / 256 for every finite code c: the exponent fields of
// the two formats differ by 8 and an e4m3 subnormal lands on an fp16 subnormal
// with the same ratio; the product by 256 is exact.  (The two NaN codes, which
// the append never writes, read as +-480.)
__device__ __forceinline__ uint4 e4m3x8_to_f16x8(uint2 v) {
  const __half2 k256 = __float2half2_rn(256.f);
  auto cvt = [&](uint32_t four, int sel) -> uint32_t {
    const uint32_t x = __byte_perm(four, 0u, sel);          // two codes in the low bytes of the halves
    const uint32_t bits = ((x & 0x007f007fu) << 7) | ((x & 0x00800080u) << 8);
    const __half2 h = __hmul2(*reinterpret_cast<const __half2*>(&bits), k256);
    return *reinterpret_cast<const uint32_t*>(&h);
  };
  return make_uint4(cvt(v.x, 0x4140), cvt(v.x, 0x4342), cvt(v.y, 0x4140), cvt(v.y, 0x4342));
}

// Two bf16 values (one word) to two fp16 values: the absorbed query of an e4m3
// decode enters the fp16 contraction.
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w) {
  const float lo = __uint_as_float(w << 16), hi = __uint_as_float(w & 0xffff0000u);
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Threads per CTA: 12 warps.  Warps 8..11 are a second softmax warpgroup with a
// bf16 cache and the e4m3 converters with an e4m3 cache.
template <bool kFp8>
constexpr int threads() { return 384; }

template <bool kFp8>
__global__ void __launch_bounds__(threads<kFp8>(), 1) __cluster_dims__(2, 1, 1)
    decode_umma_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                       const __grid_constant__ CUtensorMap qmap, const DecodeArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sb = ptx::smem_u32(smem);
  const uint32_t rank = ptx::cluster_rank();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile uint32_t* misc = reinterpret_cast<volatile uint32_t*>(smem + kOffMisc);
  auto bar = [&](int i) -> uint32_t { return sb + kOffBar + 8u * static_cast<uint32_t>(i); };
  const uint32_t iters = a.wait_limit;

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

  // set-up that reads none of the call's inputs runs before the wait for the
  // previous kernel of the stream (programmatic dependent launch)
  if (threadIdx.x == 0) {
    for (int i = 0; i < kSlots; ++i) {
      ptx::mbar_init(bar(kFull + i), 1);
      ptx::mbar_init(bar(kEmpty + i), 1);
      ptx::mbar_init(bar(kCvtDone + i), 128);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(bar(kSFull + i), 1);
      ptx::mbar_init(bar(kSEmpty + i), 128);
      ptx::mbar_init(bar(kPVDone + i), 1);
      ptx::mbar_init(bar(kStgFull + i), 128);
      ptx::mbar_init(bar(kStgFree + i), 128);
    }
    for (int i = 0; i < kPBufs; ++i) {
      ptx::mbar_init(bar(kPFull + i), 1);
      ptx::mbar_init(bar(kPBufFree + i), 1);
    }
    for (int i = 0; i < kScaleRing; ++i) ptx::mbar_init(bar(kScl + i), 128);
    ptx::mbar_init(bar(kQReady), kFp8 ? 128 : 256);
    for (int i = 0; i < kVStages; ++i) {
      ptx::mbar_init(bar(kVFull + i), 1);
      ptx::mbar_init(bar(kVEmpty + i), 1);
      ptx::mbar_init(bar(kVCvt + i), 128);
    }
    ptx::mbar_init(bar(kCorrReq), 1);
    ptx::mbar_init(bar(kCorrDone), kFp8 ? 128 : 256);
    ptx::mbar_init(bar(kOFull), 1);
    ptx::mbar_init(bar(kFin), 128);
    ptx::mbar_init(bar(kDrain), 1);
    ptx::mbar_init(bar(kDrain2), 1);
    ptx::mbar_init(bar(kCvtLd), 128);
    misc[1] = 0u;
    misc[2] = 0u;
    misc[3] = 0u;
    misc[4] = 0u;
    misc[5] = 0u;
    ptx::fence_mbar_init_cluster();
  }
  __syncwarp();
  if (warp == 1) {
    ptx::tmem_alloc(sb + kOffMisc, kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::cluster_sync();       // the peer's barriers exist before any remote arrive
  ptx::tc_fence_after();
  const uint32_t tmem = misc[0];

  grid_dep_wait();
  grid_dep_trigger();
  int bad_len = 0;
  const Split sp = split_of(a, static_cast<int>(blockIdx.x >> 1), &bad_len);
  if (bad_len && threadIdx.x == 0 && rank == 0) report_error(a.err, MLA_ERR_BAD_INDEX);
  // this split's page table, kept in shared memory
  int* table = reinterpret_cast<int*>(smem + (rank == 0 ? kOffTable0 : kOffTable1));
  for (int t = threadIdx.x; t < min(sp.ntiles, kMaxTablePages); t += blockDim.x) {
    const int pg = load_page(a, sp, t);
    table[t] = pg;
    if (pg < 0 && rank == 0) report_error(a.err, MLA_ERR_BAD_INDEX);
  }
  __syncthreads();

  if (rank == 0) {
    // =========================== CTA 0: scores and softmax ===========================
    // Slot use n = 0, 1 carries Q half n; use n >= 2 carries tile t = n - 2.
    if (warp == 0) {
      if (lane == 0) {
        // TMA producer over the ring: 2 halves of Q, then one request per page,
        // each as soon as the slot is free (its previous page's MMAs are done).
        if (!kFp8) ptx::prefetch_tmap(&kmap);
        ptx::prefetch_tmap(&qmap);
        const int total = kQLoads + sp.ntiles;
        int issued = 0;
        for (int n = 0; n < total; ++n) {
          const int slot = n % kSlots;
          if (!wait_local(bar(kEmpty + slot), ((n / kSlots) & 1) ^ 1)) break;
          const uint32_t dst = sb + kOffRing + slot * kSlotBytes;
          if (n < kQLoads) {
            ptx::mbar_arrive_expect_tx(bar(kFull + slot), kSlotBytes);
            ptx::tma_load_3d(dst, &qmap, bar(kFull + slot), 0, sp.b * kH + 64 * n, 0);
          } else {
            const int t = n - kQLoads;
            const int pg = max(page_at(a, sp, table, t), 0);
            if (kFp8) {
              // the page's codes (contiguous) into the slot's upper half, its scales
              // into scale-ring entry t % 6
              ptx::mbar_arrive_expect_tx(bar(kFull + slot), kPageF8Bytes + kScaleBytes);
              ptx::bulk_load(dst + kF8InSlot, static_cast<const uint8_t*>(a.cache) + static_cast<long>(pg) * kPageF8Bytes,
                             kPageF8Bytes, bar(kFull + slot));
              ptx::bulk_load(sb + kOffScale + (t % kScaleRing) * kScaleBytes,
                             a.cache_scale + static_cast<long>(pg) * kTok, kScaleBytes, bar(kFull + slot));
            } else {
              ptx::mbar_arrive_expect_tx(bar(kFull + slot), kSlotBytes);
              ptx::tma_load_3d(dst, &kmap, bar(kFull + slot), 0, pg * kTok, 0);
            }
          }
          issued = n + 1;
        }
        for (int n = max(0, issued - kSlots); n < issued; ++n)
          drain(bar(kFull + n % kSlots), (n / kSlots) & 1);
      }
      __syncwarp();
    } else if (warp == 1 || warp == 3) {
      // two MMA issuers, warp 1 for even tiles and warp 3 for odd ones (one S
      // buffer each): two independent streams of N = 64 MMAs keep the tensor
      // core about twice as busy as one (measured).  S[i] = Q K^T, A = Q from
      // TMEM, B = the page's chunks in the ring.
      const int w = warp == 1 ? 0 : 1;
      if (lane == 0) {
        constexpr uint32_t idS = ptx::idesc_f16_f32(128, kTok, false, false, kFp8);
        if (wait_local(bar(kQReady), 0)) {
          if (w == 0)
            for (int n = 0; n < kQLoads; ++n) ptx::mbar_arrive(bar(kEmpty + n));   // Q is in TMEM
#pragma unroll 1
          for (int t = w; t < sp.ntiles; t += 2) {
            const int i = t & 1;
            const int n = kQLoads + t;
            const int slot = n % kSlots;
            if (!wait_local(bar(kSEmpty + i), ((t >> 1) & 1) ^ 1)) break;
            // the page as an operand: as landed, or once the converters have expanded its codes
            if (!(kFp8 ? wait_local(bar(kCvtDone + slot), (t / kSlots) & 1)
                       : wait_local(bar(kFull + slot), (n / kSlots) & 1)))
              break;
            ptx::tc_fence_after();
            // S[i] = Q K^T over the 9 chunks of K = 576, one page (N = 64) per MMA
            const uint32_t d = tmem + kColS + 64u * i;
            const uint32_t kb = sb + kOffRing + slot * kSlotBytes;
#pragma unroll 3
            for (int c = 0; c < kKBoxes; ++c) {
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const uint64_t bd = ptx::sdesc_sw128(kb + c * kChunkInSlot + j * 32, 16, 1024);
                ptx::umma_ts(d, tmem + kColQ + 32u * c + 8u * j, bd, idS, (c | j) ? 1u : 0u);
              }
            }
            ptx::umma_commit(bar(kSFull + i));
            ptx::umma_commit(bar(kEmpty + slot));   // the page has been read: its slot is free
          }
        }
        ptx::umma_commit(bar(w == 0 ? kDrain : kDrain2));
        drain(bar(w == 0 ? kDrain : kDrain2), 0);
      }
      __syncwarp();
    } else if (!kFp8 && warp >= 8) {
      // bf16 cache, senders (one warp per TMEM lane quadrant): help move Q into
      // TMEM, then for every tile take the P rows the softmax staged in TMEM, with
      // the rescale factors and flags it staged in shared memory, and send them to
      // CTA 1's buffer t % 3 by asynchronous stores counted on its barrier, once
      // P V(t - 3) has read that buffer.  A transfer between the two SMs costs
      // ~0.8 us per tile this way; here it overlaps the next tile's softmax.
      const int q = warp & 3;
      const int r = q * 32 + lane;
      const uint32_t lb = static_cast<uint32_t>(q * 32) << 16;
      bool ok = wait_local(bar(kFull + (q >> 1)), 0);
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        const int row = r & 63;
        const uint8_t* base = smem + kOffRing + (q >> 1) * kSlotBytes + row * 128;
#pragma unroll 1
        for (int c = 5; c < kKBoxes; ++c) {
          uint32_t v[32];
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            const uint4 u = *reinterpret_cast<const uint4*>(base + c * kChunkInSlot + ((ch ^ (row & 7)) << 4));
            v[4 * ch] = u.x;
            v[4 * ch + 1] = u.y;
            v[4 * ch + 2] = u.z;
            v[4 * ch + 3] = u.w;
          }
          ptx::tmem_st32(tmem + lb + kColQ + 32u * c, v);
        }
      }
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      ptx::mbar_arrive(bar(kQReady));

      const uint32_t rP = ptx::mapa(sb + kOffP, 1);
      const uint32_t rPFull = ptx::mapa(bar(kPFull), 1);
      const float* astg = reinterpret_cast<const float*>(smem + kOffStg);
      const uint32_t* fstg = reinterpret_cast<const uint32_t*>(smem + kOffStg + 2 * kH * 4);
      uint32_t sent = 0;
#pragma unroll 1
      for (int t = 0; t < sp.ntiles && ok; ++t) {
        const int i = t & 1;
        bool w = wait_local(bar(kStgFull + i), (t >> 1) & 1);
        if (!__all_sync(0xffffffffu, w)) break;
        ptx::tc_fence_after();
        uint32_t v[32];
        ptx::tmem_ld32(tmem + lb + kColStg + 32u * i, v);
        ptx::tmem_wait_ld();
        const uint32_t alpha = __float_as_uint(astg[i * kH + r]);
        const uint32_t flag = fstg[i * 4 + q];
        ptx::tc_fence_before();
        ptx::mbar_arrive(bar(kStgFree + i));
        w = wait_remote(bar(kPBufFree + t % kPBufs), ((t / kPBufs) & 1) ^ 1);
        if (!__all_sync(0xffffffffu, w)) break;
        const uint32_t pbuf = rP + (t % kPBufs) * kPBufStride;
        const uint32_t pfull = rPFull + 8u * (t % kPBufs);
#pragma unroll
        for (int c = 0; c < 8; ++c)
          ptx::st_async_v4(pbuf + r * 128 + ((c ^ (r & 7)) << 4), v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3],
                           pfull);
        ptx::st_async_u32(pbuf + kPBytes + r * 4, alpha, pfull);
        if (lane == 0) ptx::st_async_u32(pbuf + kPBytes + kH * 4 + q * 4, flag, pfull);
        if (r == 0) ++sent;
      }
      if (r == 0) ptx::st_cluster_u32(ptx::mapa(sb + kOffMisc + 12, 1), sent);
    } else if (!kFp8 && warp >= 4) {
      // bf16 cache, softmax warpgroup (thread = head row r, TMEM lane quadrant q):
      // the online softmax of every tile, its P row staged in TMEM and the
      // rescale factor / flag in shared memory for the senders
      const int q = warp & 3;
      const int r = q * 32 + lane;
      const uint32_t lb = static_cast<uint32_t>(q * 32) << 16;
      bool ok = wait_local(bar(kFull + (q >> 1)), 0);
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        const int row = r & 63;
        const uint8_t* base = smem + kOffRing + (q >> 1) * kSlotBytes + row * 128;
#pragma unroll 1
        for (int c = 0; c < 5; ++c) {
          uint32_t v[32];
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            const uint4 u = *reinterpret_cast<const uint4*>(base + c * kChunkInSlot + ((ch ^ (row & 7)) << 4));
            v[4 * ch] = u.x;
            v[4 * ch + 1] = u.y;
            v[4 * ch + 2] = u.z;
            v[4 * ch + 3] = u.w;
          }
          ptx::tmem_st32(tmem + lb + kColQ + 32u * c, v);
        }
      }
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      ptx::mbar_arrive(bar(kQReady));

      const uint32_t rL = ptx::mapa(sb + kOffLfin, 1);
      const uint32_t rFin = ptx::mapa(bar(kFin), 1);
      float* astg = reinterpret_cast<float*>(smem + kOffStg);
      uint32_t* fstg = reinterpret_cast<uint32_t*>(smem + kOffStg + 2 * kH * 4);
      const float sl2 = a.scale * kLog2e;
      float m_used = -INFINITY, l = 0.f;
#pragma unroll 1
      for (int t = 0; t < sp.ntiles && ok; ++t) {
        const int i = t & 1;
        bool w = wait_local(bar(kSFull + i), (t >> 1) & 1);
        if (!__all_sync(0xffffffffu, w)) break;
        ptx::tc_fence_after();
        uint32_t s0[32], s1[32];
        ptx::tmem_ld32(tmem + lb + kColS + 64u * i, s0);
        ptx::tmem_ld32(tmem + lb + kColS + 64u * i + 32u, s1);
        ptx::tmem_wait_ld();
        ptx::tc_fence_before();
        ptx::mbar_arrive(bar(kSEmpty + i));
        const int valid = valid_tokens(sp, page_at(a, sp, table, t), t);
        // tile max on the raw scores (the scale is positive), then one FFMA per
        // exponent: p_j = 2^(s_j * scale * log2(e) - m); masking only on a ragged tile
        if (valid < kTok) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            if (j >= valid) s0[j] = __float_as_uint(-INFINITY);
            if (j + 32 >= valid) s1[j] = __float_as_uint(-INFINITY);
          }
        }
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int j = 0; j < 32; ++j)
          mx[j & 3] = fmaxf(mx[j & 3], fmaxf(__uint_as_float(s0[j]), __uint_as_float(s1[j])));
        const float m_tile = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * sl2;
        const bool resc = m_tile > m_used + kRescaleThreshold;
        float alpha = 1.f;
        if (resc) {
          alpha = (m_used == -INFINITY) ? 0.f : ptx::ex2(m_used - m_tile);
          m_used = m_tile;
        }
        uint32_t pk[32];
        float psum = 0.f;
        if (m_used != -INFINITY) {
          const float nm = -m_used;
          float ps[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float p0 = ptx::ex2(fmaf(__uint_as_float(s0[2 * j]), sl2, nm));
            const float p1 = ptx::ex2(fmaf(__uint_as_float(s0[2 * j + 1]), sl2, nm));
            const float p2 = ptx::ex2(fmaf(__uint_as_float(s1[2 * j]), sl2, nm));
            const float p3 = ptx::ex2(fmaf(__uint_as_float(s1[2 * j + 1]), sl2, nm));
            ps[j & 3] += (p0 + p1) + (p2 + p3);
            const __nv_bfloat162 pa = __floats2bfloat162_rn(p0, p1), pb = __floats2bfloat162_rn(p2, p3);
            pk[j] = *reinterpret_cast<const uint32_t*>(&pa);
            pk[j + 16] = *reinterpret_cast<const uint32_t*>(&pb);
          }
          psum = (ps[0] + ps[1]) + (ps[2] + ps[3]);
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) pk[j] = 0u;
        }
        l = l * alpha + psum;
        // stage: P row in TMEM buffer t & 1, alpha and the warp's rescale flag in
        // shared memory, once the senders have taken tile t - 2 out of them
        w = wait_local(bar(kStgFree + i), ((t >> 1) & 1) ^ 1);
        if (!__all_sync(0xffffffffu, w)) break;
        ptx::tc_fence_after();
        ptx::tmem_st32(tmem + lb + kColStg + 32u * i, pk);
        astg[i * kH + r] = alpha;
        const unsigned any = __any_sync(0xffffffffu, resc && t > 0);
        if (lane == 0) fstg[i * 4 + q] = any;
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        ptx::mbar_arrive(bar(kStgFull + i));
      }
      // this split's log-sum-exp (natural log) and the normaliser for CTA 1
      const long row = (static_cast<long>(sp.b) * a.num_splits + sp.split) * kH + r;
      a.lse_part[row] = l > 0.f ? (m_used + log2f(l)) * kLn2 : -INFINITY;
      ptx::st_cluster_u32(rL + r * 4, __float_as_uint(l));
      ptx::mbar_arrive_remote(rFin);
    } else if (warp >= 4 && warp < 8) {
      // softmax warpgroup: thread = head row r, TMEM lane quadrant q
      const int q = warp & 3;
      const int r = q * 32 + lane;
      const uint32_t lb = static_cast<uint32_t>(q * 32) << 16;
      // Q half q/2 (ring slot q/2) holds this warp's 32 heads as 9 column chunks
      // of 64 rows; the MMA warp frees the slots once every thread has arrived
      // on q_ready.  An e4m3 decode contracts in fp16: Q is converted here.
      bool ok = wait_local(bar(kFull + (q >> 1)), 0);
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        const int row = r & 63;
        const uint8_t* base = smem + kOffRing + (q >> 1) * kSlotBytes + row * 128;
#pragma unroll 1
        for (int c = 0; c < kKBoxes; ++c) {
          uint32_t v[32];
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            const uint4 u = *reinterpret_cast<const uint4*>(base + c * kChunkInSlot + ((ch ^ (row & 7)) << 4));
            v[4 * ch] = u.x;
            v[4 * ch + 1] = u.y;
            v[4 * ch + 2] = u.z;
            v[4 * ch + 3] = u.w;
          }
          if (kFp8) {
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = bf16x2_to_f16x2(v[e]);
          }
          ptx::tmem_st32(tmem + lb + kColQ + 32u * c, v);
        }
      }
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      ptx::mbar_arrive(bar(kQReady));

      const uint32_t rP = ptx::mapa(sb + kOffP, 1);    // CTA 1's P buffers
      const uint32_t rL = ptx::mapa(sb + kOffLfin, 1);
      const uint32_t rPFull = ptx::mapa(bar(kPFull), 1);
      const uint32_t rFin = ptx::mapa(bar(kFin), 1);
      const float sl2 = a.scale * kLog2e;
      float m_used = -INFINITY, l = 0.f;
      uint32_t sent = 0;
#pragma unroll 1
      for (int t = 0; t < sp.ntiles && ok; ++t) {
        const int i = t & 1;
        bool w = wait_local(bar(kSFull + i), (t >> 1) & 1);
        if (!__all_sync(0xffffffffu, w)) break;
        ptx::tc_fence_after();
        uint32_t s0[32], s1[32];
        ptx::tmem_ld32(tmem + lb + kColS + 64u * i, s0);
        ptx::tmem_ld32(tmem + lb + kColS + 64u * i + 32u, s1);
        ptx::tmem_wait_ld();
        ptx::tc_fence_before();
        ptx::mbar_arrive(bar(kSEmpty + i));
        const int valid = valid_tokens(sp, page_at(a, sp, table, t), t);
        // e4m3 cache: row j is scale_j times its codes, so score j is scale_j times
        // the score against the codes (the converters pass on the landed scales)
        const float* scl = reinterpret_cast<const float*>(smem + kOffScale + (t % kScaleRing) * kScaleBytes);
        if (kFp8) {
          w = wait_local(bar(kScl + t % kScaleRing), (t / kScaleRing) & 1);
          if (!__all_sync(0xffffffffu, w)) break;
        }
        uint32_t pk[32];
        float psum = 0.f;
        float alpha = 1.f;
        bool resc = false;
        if constexpr (!kFp8) {
          // tile max on the raw scores (the scale is positive), then one FFMA per
          // exponent: p_j = 2^(s_j * scale * log2(e) - m); masking only on a ragged tile
          if (valid < kTok) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              if (j >= valid) s0[j] = __float_as_uint(-INFINITY);
              if (j + 32 >= valid) s1[j] = __float_as_uint(-INFINITY);
            }
          }
          float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int j = 0; j < 32; ++j)
            mx[j & 3] = fmaxf(mx[j & 3], fmaxf(__uint_as_float(s0[j]), __uint_as_float(s1[j])));
          const float m_tile = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * sl2;
          resc = m_tile > m_used + kRescaleThreshold;
          if (resc) {
            alpha = (m_used == -INFINITY) ? 0.f : ptx::ex2(m_used - m_tile);
            m_used = m_tile;
          }
          if (m_used != -INFINITY) {
            const float nm = -m_used;
            float ps[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const float p0 = ptx::ex2(fmaf(__uint_as_float(s0[2 * j]), sl2, nm));
              const float p1 = ptx::ex2(fmaf(__uint_as_float(s0[2 * j + 1]), sl2, nm));
              const float p2 = ptx::ex2(fmaf(__uint_as_float(s1[2 * j]), sl2, nm));
              const float p3 = ptx::ex2(fmaf(__uint_as_float(s1[2 * j + 1]), sl2, nm));
              ps[j & 3] += (p0 + p1) + (p2 + p3);
              const __nv_bfloat162 pa = __floats2bfloat162_rn(p0, p1), pb = __floats2bfloat162_rn(p2, p3);
              pk[j] = *reinterpret_cast<const uint32_t*>(&pa);
              pk[j + 16] = *reinterpret_cast<const uint32_t*>(&pb);
            }
            psum = (ps[0] + ps[1]) + (ps[2] + ps[3]);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) pk[j] = 0u;
          }
        } else {
          float x[64];
          float m_tile = -INFINITY;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float f0 = sl2 * scl[j], f1 = sl2 * scl[j + 32];
            x[j] = j < valid ? __uint_as_float(s0[j]) * f0 : -INFINITY;
            x[j + 32] = j + 32 < valid ? __uint_as_float(s1[j]) * f1 : -INFINITY;
            m_tile = fmaxf(m_tile, fmaxf(x[j], x[j + 32]));
          }
          resc = m_tile > m_used + kRescaleThreshold;
          if (resc) {
            alpha = (m_used == -INFINITY) ? 0.f : ptx::ex2(m_used - m_tile);
            m_used = m_tile;
          }
          const bool live = m_used != -INFINITY;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float p0 = live ? ptx::ex2(x[2 * j] - m_used) : 0.f;
            const float p1 = live ? ptx::ex2(x[2 * j + 1] - m_used) : 0.f;
            // the P V operand carries scale_j (V holds the codes); l sums the weights
            psum += p0 + p1;
            const __half2 ph = __floats2half2_rn(2 * j < valid ? p0 * scl[2 * j] : 0.f,
                                                 2 * j + 1 < valid ? p1 * scl[2 * j + 1] : 0.f);
            pk[j] = *reinterpret_cast<const uint32_t*>(&ph);
          }
        }
        l = l * alpha + psum;
        // row r of P(t), its rescale factor and (lane 0) the warp's rescale flag go
        // to CTA 1's buffer t % 3 by asynchronous stores counted on its barrier,
        // once P V(t - 3) has finished reading that buffer
        w = wait_remote(bar(kPBufFree + t % kPBufs), ((t / kPBufs) & 1) ^ 1);
        if (!__all_sync(0xffffffffu, w)) break;
        const uint32_t pbuf = rP + (t % kPBufs) * kPBufStride;
        const uint32_t pfull = rPFull + 8u * (t % kPBufs);
#pragma unroll
        for (int c = 0; c < 8; ++c)
          ptx::st_async_v4(pbuf + r * 128 + ((c ^ (r & 7)) << 4), pk[4 * c], pk[4 * c + 1], pk[4 * c + 2],
                           pk[4 * c + 3], pfull);
        ptx::st_async_u32(pbuf + kPBytes + r * 4, __float_as_uint(alpha), pfull);
        const unsigned any = __any_sync(0xffffffffu, resc && t > 0);
        if (lane == 0) ptx::st_async_u32(pbuf + kPBytes + kH * 4 + q * 4, any, pfull);
        if (r == 0) ++sent;
      }
      // this split's log-sum-exp (natural log) and the normaliser for CTA 1
      const long row = (static_cast<long>(sp.b) * a.num_splits + sp.split) * kH + r;
      a.lse_part[row] = l > 0.f ? (m_used + log2f(l)) * kLn2 : -INFINITY;
      ptx::st_cluster_u32(rL + r * 4, __float_as_uint(l));
      ptx::mbar_arrive_remote(rFin);
      if (r == 0) ptx::st_cluster_u32(ptx::mapa(sb + kOffMisc + 12, 1), sent);
    } else if (kFp8 && warp >= 8) {
      // converters: expand a landed page's e4m3 codes, in place, into the fp16
      // chunk-major swizzled layout S = Q K^T reads, and pass the page's scales on
      // to the softmax.  Every thread holds its share of the codes in registers
      // before any thread writes (the fp16 page covers the codes' bytes).
      const int ct = static_cast<int>(threadIdx.x) - 256;
#pragma unroll 1
      for (int t = 0; t < sp.ntiles; ++t) {
        const int n = kQLoads + t, slot = n % kSlots;
        bool ok = wait_local(bar(kFull + slot), (n / kSlots) & 1);
        if (!__all_sync(0xffffffffu, ok)) break;
        ptx::mbar_arrive(bar(kScl + t % kScaleRing));
        uint8_t* page = smem + kOffRing + slot * kSlotBytes;
        uint2 u[kF8UnitsK];
#pragma unroll
        for (int k = 0; k < kF8UnitsK; ++k)
          u[k] = *reinterpret_cast<const uint2*>(page + kF8InSlot + (k * 128 + ct) * 8);
        ptx::mbar_arrive(bar(kCvtLd));
        ok = wait_local(bar(kCvtLd), t & 1);
        if (!__all_sync(0xffffffffu, ok)) break;
#pragma unroll
        for (int k = 0; k < kF8UnitsK; ++k) {
          const int g = k * 128 + ct, row = g / 72, cu = g - row * 72;
          *reinterpret_cast<uint4*>(page + (cu >> 3) * kChunkInSlot + row * 128 + (((cu & 7) ^ (row & 7)) << 4)) =
              e4m3x8_to_f16x8(u[k]);
        }
        ptx::fence_proxy_async_cta();              // generic writes -> tensor-core reads
        ptx::mbar_arrive(bar(kCvtDone + slot));
      }
    }
  } else {
    // =========================== CTA 1: values ===========================
    if (warp == 0) {
      if (lane == 0) {
        // TMA producer: first 512 columns of the same pages
        if (!kFp8) ptx::prefetch_tmap(&vmap);
        int issued = 0;
        for (int t = 0; t < sp.ntiles; ++t) {
          const int st = t % kVStages;
          if (!wait_local(bar(kVEmpty + st), ((t / kVStages) & 1) ^ 1)) break;
          const int pg = max(page_at(a, sp, table, t), 0);
          if (kFp8) {
            ptx::mbar_arrive_expect_tx(bar(kVFull + st), kPageF8Bytes);
            ptx::bulk_load(sb + kOffV + st * kVStageBytes + kF8InStage,
                           static_cast<const uint8_t*>(a.cache) + static_cast<long>(pg) * kPageF8Bytes,
                           kPageF8Bytes, bar(kVFull + st));
          } else {
            ptx::mbar_arrive_expect_tx(bar(kVFull + st), kVStageBytes);
            ptx::tma_load_3d(sb + kOffV + st * kVStageBytes, &vmap, bar(kVFull + st), 0, pg * kTok, 0);
          }
          issued = t + 1;
        }
        for (int t = max(0, issued - kVStages); t < issued; ++t)
          drain(bar(kVFull + t % kVStages), (t / kVStages) & 1);
      }
      __syncwarp();
    } else if (warp == 1) {
      // MMA issuer: O += P V  (A = P, K-major; B = V, MN-major; two N = 256 halves)
      constexpr uint32_t idPV = ptx::idesc_f16_f32(128, 256, false, true, kFp8);
      int ncorr = 0;
#pragma unroll 1
      for (int t = 0; t < sp.ntiles; ++t) {
        const int st = t & 1, pbi = t % kPBufs;
        bool ok = wait_local(bar((kFp8 ? kVCvt : kVFull) + st), (t >> 1) & 1);
        ok = ok && wait_remote(bar(kPFull + pbi), (t / kPBufs) & 1);
        if (!__all_sync(0xffffffffu, ok)) break;
        ptx::fence_proxy_async_cta();   // P arrived by asynchronous stores: order it before the MMAs' reads
        const int valid = valid_tokens(sp, page_at(a, sp, table, t), t);
        if (!kFp8 && valid < kTok) {
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
        const uint8_t* msg = smem + kOffP + pbi * kPBufStride;
        const uint32_t* fl = reinterpret_cast<const uint32_t*>(msg + kPBytes + kH * 4);
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
          const uint32_t pb = sb + kOffP + pbi * kPBufStride;
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
    } else if (warp == 2) {
      // release: a finished P V frees its V stage and its P buffer (CTA 0 waits
      // for the latter before sending the next tile's P into it)
      if (lane == 0) {
        const uint32_t rPBufFree = ptx::mapa(bar(kPBufFree), 0);
        for (int t = 0; t < sp.ntiles; ++t) {
          const int i = t & 1;
          if (!wait_local(bar(kPVDone + i), (t >> 1) & 1)) break;
          ptx::mbar_arrive(bar(kVEmpty + i));
          ptx::mbar_arrive_remote(rPBufFree + 8u * (t % kPBufs));
        }
      }
      __syncwarp();
    } else if (warp == 3) {
      // P receiver: arms each tile's P barrier with the bytes the softmax sends
      // (16,912) and follows its completion, so that the teardown knows what is
      // still in flight after a failed wait
      if (lane == 0) {
        for (int t = 0; t < sp.ntiles; ++t) {
          const int pbi = t % kPBufs;
          ptx::mbar_arrive_expect_tx(bar(kPFull + pbi), kPMsgBytes);
          misc[5] = static_cast<uint32_t>(t + 1);
          if (!wait_remote(bar(kPFull + pbi), (t / kPBufs) & 1)) break;
          misc[4] = static_cast<uint32_t>(t + 1);
        }
      }
      __syncwarp();
    } else if (warp >= 4 && (warp < 8 || !kFp8)) {
      // correction (rescale O rows on request) and epilogue; with a bf16 cache two
      // warpgroups share them, warps 4..7 taking O's columns 0..255 and warps 8..11
      // columns 256..511
      constexpr int kGroups = kFp8 ? 1 : 2;
      const int wg = warp >> 3;
      const int c0 = wg * (16 / kGroups), c1 = c0 + 16 / kGroups;    // 32-column blocks of O
      const int q = warp & 3;
      const int r = q * 32 + lane;
      const uint32_t lb = static_cast<uint32_t>(q * 32) << 16;
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
        const float al =
            reinterpret_cast<const float*>(smem + kOffP + (t % kPBufs) * kPBufStride + kPBytes)[r];
#pragma unroll 1
        for (int c = c0; c < c1; ++c) {
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
      // o_part[b][split][c/8][h][c%8] in fp16: per group of eight columns the 32
      // lanes store 32 consecutive heads' 16 bytes (512 contiguous bytes)
      uint4* obase = reinterpret_cast<uint4*>(a.o_part) +
                     (static_cast<long>(sp.b) * a.num_splits + sp.split) * (kDc / 8) * kH + r;
      if (ok) {
        ptx::tc_fence_after();
        const float lsum = reinterpret_cast<const volatile float*>(smem + kOffLfin)[r];
        const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
        float big = 0.f;
        if (sp.ntiles == 0) {
          for (int g = 4 * c0; g < 4 * c1; ++g) obase[g * kH] = make_uint4(0u, 0u, 0u, 0u);
        } else {
          // two 32-column blocks per TMEM round trip where registers allow (bf16)
          constexpr int kPer = kFp8 ? 1 : 2;
#pragma unroll 1
          for (int c = c0; c < c1; c += kPer) {
            uint32_t v[kPer][32];
#pragma unroll
            for (int j = 0; j < kPer; ++j) ptx::tmem_ld32(tmem + lb + kColO + 32u * (c + j), v[j]);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < kPer; ++j)
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                uint32_t hw[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                  const float x0 = __uint_as_float(v[j][8 * e + 2 * k]) * inv;
                  const float x1 = __uint_as_float(v[j][8 * e + 2 * k + 1]) * inv;
                  big = fmaxf(big, fmaxf(fabsf(x0), fabsf(x1)));
                  const __half2 hh = __floats2half2_rn(x0, x1);
                  hw[k] = *reinterpret_cast<const uint32_t*>(&hh);
                }
                obase[(4 * (c + j) + e) * kH] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
              }
          }
        }
        // fp16 holds |x| <= 65504 (the largest finite value); beyond it the
        // partial would be infinite
        if (!(big <= 65504.f)) report_error(a.err, MLA_ERR_RANGE);
        ptx::tc_fence_before();
      }
    } else if (kFp8 && warp >= 8) {
      // converters: the first 512 columns of a landed page to fp16, in place, in
      // the stage's chunk-major swizzled layout (the MN-major V operand); rows past
      // the sequence end become zeros so that P = 0 meets finite V
      const int ct = static_cast<int>(threadIdx.x) - 256;
#pragma unroll 1
      for (int t = 0; t < sp.ntiles; ++t) {
        const int st = t % kVStages;
        bool ok = wait_local(bar(kVFull + st), (t / kVStages) & 1);
        if (!__all_sync(0xffffffffu, ok)) break;
        const int valid = valid_tokens(sp, page_at(a, sp, table, t), t);
        uint8_t* stage = smem + kOffV + st * kVStageBytes;
        uint2 u[kF8UnitsV];
#pragma unroll
        for (int k = 0; k < kF8UnitsV; ++k) {
          const int g = k * 128 + ct, row = g >> 6, cu = g & 63;
          u[k] = row < valid ? *reinterpret_cast<const uint2*>(stage + kF8InStage + row * kD + cu * 8)
                             : make_uint2(0u, 0u);
        }
        ptx::mbar_arrive(bar(kCvtLd));
        ok = wait_local(bar(kCvtLd), t & 1);
        if (!__all_sync(0xffffffffu, ok)) break;
#pragma unroll
        for (int k = 0; k < kF8UnitsV; ++k) {
          const int g = k * 128 + ct, row = g >> 6, cu = g & 63;
          *reinterpret_cast<uint4*>(stage + (cu >> 3) * kBoxBytes + row * 128 + (((cu & 7) ^ (row & 7)) << 4)) =
              e4m3x8_to_f16x8(u[k]);
        }
        ptx::fence_proxy_async_cta();
        ptx::mbar_arrive(bar(kVCvt + st));
      }
    }
  }

  __syncwarp();
  __syncthreads();
  ptx::cluster_sync();       // CTA 1 now sees how many P messages CTA 0 sent
  if (rank == 1 && threadIdx.x == 0) {
    // after a wait gave up, stores may still be landing: arm and await each tile
    // not consumed yet (in order, so that phase parities stay in step)
    const uint32_t sent = misc[3], armed = misc[5];
    for (uint32_t t = misc[4]; t < sent; ++t) {
      if (t >= armed) ptx::mbar_arrive_expect_tx(bar(kPFull + t % kPBufs), kPMsgBytes);
      drain(bar(kPFull + t % kPBufs), (t / kPBufs) & 1);
    }
  }
  __syncwarp();
  __syncthreads();
  ptx::cluster_sync();       // no copy in flight and no remote access after this point
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace dec
}  // namespace mla

// Weight-streaming GEMM on tcgen05 tensor cores for the projections around
// the decode (batch of B <= 256 decode tokens against large bf16 weights):
//
//   D[m][b] = sum_k A[m][k] * X[b][k]
//
// with the weight as the M operand (128 rows per tile, "swap-AB": the batch
// is the N dimension, 16 <= N <= 256) and fp32 accumulation in TMEM.  Uses:
//   * W_O   (V2 page section 2.3, W_UV absorbed into W_O; applied as W_O after
//            W_UV):  A = W_O [5120][16384] K-major, X = o [B][16384];
//            stream-K: the grid's CTAs (one per SM) share the (M tile, K box)
//            stages evenly, each writing one fp32 partial tile per M tile it
//            touches; a second kernel sums them in a fixed order.
//   * W_UV  per head:  A = W_UV[h] [128][512] K-major, X = o_lat[:, h, :].
//   * W_UK  per head (absorbed query, V2 page section 2.3):  A = W_UK[h]^T,
//            i.e. W_UK[h] [128][512] read MN-major, X = q_nope[:, h, :];
//            the epilogue also applies RoPE to q_pe (section 2.2).
//
// HBM-bound on the weight stream (2 flops per weight byte per token of the
// batch).  Each pipeline stage is ONE 3-D TMA request for A (kcs chunks of 64
// along K, landing chunk-major in the 128-byte-swizzled UMMA layout) and one
// for X, so a stage moves 16*kcs KB of weights with two requests; a CTA may
// own several consecutive M tiles of one group, each accumulating in its own
// TMEM columns.  One thread issues the UMMAs, four warps drain TMEM.
//
// The weights are no output of an earlier kernel, so the first stages' weight
// boxes are requested before the wait for the previous kernel of the stream
// (programmatic dependent launch); X and everything else come after it.
#pragma once

#include "device_common.cuh"
#include "sm100_ptx.cuh"

namespace mla {
namespace gemm {

constexpr int kM = 128;          // weight rows per tile
constexpr int kKc = 64;          // K per chunk (one 128-byte swizzle row of bf16)
constexpr uint64_t kWaitNs = 1000000000ull;

enum class Epi : int { kStoreBf16T = 0, kPartialF32 = 1, kAbsorb = 2 };

struct Params {
  int n;                 // padded batch (multiple of 16), the UMMA N
  int batch;             // real batch
  int k_chunks;          // K / 64 per group
  int k_split;           // CTAs along K (gridDim.y)
  int m_per_group;       // weight rows of one group (head), multiple of 128
  int mt_per_cta;        // M tiles of one group handled by one CTA
  int kcs;               // K chunks per pipeline stage (box depth)
  int x_chunks;          // > 0: X is loaded once per CTA (all its x_chunks K chunks,
                         // which must be the CTA's whole K range) and stays resident;
                         // the stages then carry the weight only
  // A coordinates: K-major: (elem, row = group*a_row_group + m, chunk = k/64)
  //                MN-major: (elem, row = group*a_row_group + k, chunk = m/64)
  int a_row_group;
  // X coordinates: (elem, row = b, chunk = (group*x_col_group + k)/64)
  int x_col_group;
  int stages;
  // epilogue
  void* out;             // bf16 output or fp32 partials
  long out_ld;           // elements between consecutive b
  long out_group;        // elements between consecutive groups
  long out_split;        // fp32 partials: elements between K splits
  // absorb epilogue (RoPE of q_pe into q_lat[:, h, d_c:])
  const __nv_bfloat16* q_pe;
  const int32_t* pos;
  const float2* rope_cs;
  int num_heads, d_c, d_r, max_position;
  // W_UV fed straight from split-KV partials: the resident X slice o_lat[:, h, :]
  // is merged in the kernel (log-sum-exp weights, as the merge kernel computes
  // them) instead of being loaded; comb_splits = 0 turns this off
  const __half* comb_opart;    // o_part fp16 [batch][S][d_c/8][H][8]
  const float* comb_lse;       // lse_part [batch][S][H]
  int comb_splits;             // S
  __nv_bfloat16* comb_olat;    // optional: o_lat [batch][H][d_c] is written too
  float* comb_lse_out;         // optional: lse [batch][H]
  // stream-K over one group: sk_units = (m_per_group / 128) x sk_box stages,
  // sk_box = stages per M tile; CTA c takes stages [c U / G, (c + 1) U / G) of
  // the grid's G and writes partial slot c * mt_per_cta + t for the t-th M tile
  // it touches (mt_per_cta is then the slots per CTA); sk_units = 0: off
  int sk_units;
  int sk_box;
  // K-major A stored tile by tile: [M/128][K/64][128 rows][64], so that one
  // box of kcs chunks is one contiguous run of 16*kcs KB (coordinates
  // (0, 0, tile * k_chunks + chunk)); 0: row-major
  int a_tiled;
  int* err;
  uint32_t wait_limit;
};

// Threads of the CTA that build a merged X slice (warps 2..7).
constexpr int kCombThreads = 192;

template <bool kAMn, Epi kEpi>
__global__ void __launch_bounds__(256, 1)
    gemm_wt_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmX,
                   const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sb = ptx::smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool sk = kEpi == Epi::kPartialF32 && p.sk_units > 0;   // stream-K: W_O only
  const int m_tiles = p.m_per_group / kM;
  const int cta_per_group = sk ? 1 : m_tiles / p.mt_per_cta;
  const int group = sk ? 0 : blockIdx.x / cta_per_group;
  const int mt0 = sk ? 0 : (blockIdx.x % cta_per_group) * p.mt_per_cta;
  const int split = sk ? 0 : blockIdx.y;
  const int kc0 = sk ? 0 : static_cast<int>((static_cast<long>(split) * p.k_chunks) / p.k_split);
  const int kc1 = sk ? p.k_chunks : static_cast<int>((static_cast<long>(split + 1) * p.k_chunks) / p.k_split);
  const int u0 = sk ? static_cast<int>(static_cast<long>(blockIdx.x) * p.sk_units / gridDim.x) : 0;
  const int u1 = sk ? static_cast<int>(static_cast<long>(blockIdx.x + 1) * p.sk_units / gridDim.x) : 0;
  const int nst_k = sk ? p.sk_box : (kc1 - kc0 + p.kcs - 1) / p.kcs;     // stages per M tile
  const int nst = sk ? u1 - u0 : nst_k * p.mt_per_cta;
  // accumulator blocks written: M tiles of this CTA
  const int nacc = !sk ? p.mt_per_cta : (nst > 0 ? (u1 - 1) / p.sk_box - u0 / p.sk_box + 1 : 0);
  // stage i -> M tile, first K chunk, accumulator block, and whether it starts the block
  struct StageAt {
    int mt, kc, t;
    bool first;
  };
  auto stage_at = [&](int i) -> StageAt {
    StageAt r;
    if (sk) {
      const int u = u0 + i;
      r.mt = u / p.sk_box;
      r.kc = (u % p.sk_box) * p.kcs;
      r.t = r.mt - u0 / p.sk_box;
      r.first = i == 0 || u % p.sk_box == 0;
    } else {
      r.mt = mt0 + i / nst_k;
      r.kc = kc0 + (i % nst_k) * p.kcs;
      r.t = i / nst_k;
      r.first = i % nst_k == 0;
    }
    return r;
  };

  const bool xres = p.x_chunks > 0;
  const int a_bytes = kM * kKc * 2 * p.kcs;              // 16 KB per chunk
  const int x_bytes = p.n * kKc * 2 * p.kcs;             // n rows of 128 B per chunk
  const int xres_bytes = xres ? p.n * kKc * 2 * p.x_chunks : 0;
  const int stage_bytes = a_bytes + (xres ? 0 : x_bytes);  // multiple of 1024 (n % 8 == 0)
  const uint32_t stage0 = sb + xres_bytes;               // resident X first, then the stages
  const uint32_t bars = stage0 + p.stages * stage_bytes;
  auto full = [&](int s) { return bars + 8u * s; };
  auto empty = [&](int s) { return bars + 8u * (p.stages + s); };
  const uint32_t done = bars + 8u * (2 * p.stages);
  const uint32_t drainb = done + 8u;
  const uint32_t xfull = drainb + 8u;
  const uint32_t wready = xfull + 8u;
  const bool xcomb = kEpi == Epi::kStoreBf16T && xres && p.comb_splits > 0;   // W_UV only
  volatile uint32_t* misc = reinterpret_cast<volatile uint32_t*>(smem + xres_bytes + p.stages * stage_bytes +
                                                                 8 * (2 * p.stages + 4));
  float* wts = reinterpret_cast<float*>(smem + xres_bytes + p.stages * stage_bytes + 8 * (2 * p.stages + 4) + 16);
  // TMEM: one block of ncpt columns per M tile
  const uint32_t ncpt = p.n <= 32 ? 32u : (p.n <= 64 ? 64u : (p.n <= 128 ? 128u : 256u));
  uint32_t ncols = 32;
  while (ncols < ncpt * p.mt_per_cta) ncols <<= 1;
  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      ptx::mbar_init(full(s), 1);
      ptx::mbar_init(empty(s), 1);
    }
    ptx::mbar_init(done, 1);
    ptx::mbar_init(drainb, 1);
    ptx::mbar_init(xfull, xcomb ? kCombThreads : 1);
    ptx::mbar_init(wready, kCombThreads);
    misc[1] = 0u;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncwarp();
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_u32(const_cast<uint32_t*>(misc)), ncols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = misc[0];
  if (warp != 0 || lane != 0) {
    grid_dep_wait();
    grid_dep_trigger();
  }

  auto fail = [&]() {
    misc[1] = 1u;
    report_error(p.err, MLA_ERR_TIMEOUT);
  };
  auto wait = [&](uint32_t b_, uint32_t par) -> bool {
    if (misc[1]) return false;
    const bool ok = ptx::mbar_wait<false>(b_, par, p.wait_limit, kWaitNs);
    if (!ok) fail();
    return ok;
  };

  if (warp == 0) {
    if (lane == 0) {
      ptx::prefetch_tmap(&tmA);
      ptx::prefetch_tmap(&tmX);
      auto load_a = [&](int i) {
        const StageAt st = stage_at(i);
        const uint32_t dA = stage0 + (i % p.stages) * stage_bytes;
        if (kAMn) {
          // rows = K (kcs*64 of them), chunks = two 64-wide slices of this M tile
          ptx::tma_load_3d(dA, &tmA, full(i % p.stages), 0, group * p.a_row_group + st.kc * kKc, st.mt * 2);
        } else {
          if (p.a_tiled)
            ptx::tma_load_3d(dA, &tmA, full(i % p.stages), 0, 0, st.mt * p.k_chunks + st.kc);
          else
            ptx::tma_load_3d(dA, &tmA, full(i % p.stages), 0, group * p.a_row_group + st.mt * kM, st.kc);
        }
      };
      auto load_x = [&](int i) {
        const uint32_t dX = stage0 + (i % p.stages) * stage_bytes + a_bytes;
        ptx::tma_load_3d(dX, &tmX, full(i % p.stages), 0, 0, (group * p.x_col_group) / kKc + stage_at(i).kc);
      };
      // the first stages' weights, before the wait for the previous kernel
      const int pre = min(p.stages, nst);
      for (int i = 0; i < pre; ++i) {
        ptx::mbar_arrive_expect_tx(full(i), stage_bytes);
        load_a(i);
      }
      grid_dep_wait();
      grid_dep_trigger();
      if (xres && !xcomb && nst > 0) {
        // the CTA's whole slice of X, once
        ptx::mbar_arrive_expect_tx(xfull, xres_bytes);
        ptx::tma_load_3d(sb, &tmX, xfull, 0, 0, (group * p.x_col_group) / kKc + kc0);
      }
      if (!xres)
        for (int i = 0; i < pre; ++i) load_x(i);
      int issued = pre;
      for (int i = pre; i < nst; ++i) {
        const int s = i % p.stages;
        if (!wait(empty(s), ((i / p.stages) & 1) ^ 1)) break;
        ptx::mbar_arrive_expect_tx(full(s), stage_bytes);
        load_a(i);
        if (!xres) load_x(i);
        issued = i + 1;
      }
      for (int i = max(0, issued - p.stages); i < issued; ++i)
        ptx::mbar_wait<false>(full(i % p.stages), (i / p.stages) & 1, 0xffffffffu, kWaitNs);
      if (xres && !xcomb && nst > 0) ptx::mbar_wait<false>(xfull, 0, 0xffffffffu, kWaitNs);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = ptx::idesc_bf16_f32(kM, p.n, kAMn, false);
      const bool xok = !xres || nst == 0 || wait(xfull, 0);
      for (int i = 0; i < nst && xok; ++i) {
        const int s = i % p.stages;
        if (!wait(full(s), (i / p.stages) & 1)) break;
        ptx::tc_fence_after();
        const uint32_t aB = stage0 + s * stage_bytes;
        const StageAt st = stage_at(i);
        // X chunks of this stage: in the stage, or at their place in the resident slice
        const uint32_t xB = xres ? sb + (st.kc - kc0) * (p.n * 128) : aB + a_bytes;
        const uint32_t d = tmem + ncpt * static_cast<uint32_t>(st.t);
        const int nkc = min(p.kcs, kc1 - st.kc);   // chunks of this stage in range
        for (int c = 0; c < nkc; ++c) {
#pragma unroll
          for (int j = 0; j < kKc / 16; ++j) {
            const uint64_t ad = kAMn
                ? ptx::sdesc_sw128(aB + (c * kKc + 16 * j) * 128, kKc * p.kcs * 128, 1024)
                : ptx::sdesc_sw128(aB + c * (kM * 128) + 32 * j, 16, 1024);
            const uint64_t xd = ptx::sdesc_sw128(xB + c * (p.n * 128) + 32 * j, 16, 1024);
            ptx::umma_ss(d, ad, xd, idesc, (!st.first || c > 0 || j > 0) ? 1u : 0u);
          }
        }
        ptx::umma_commit(empty(s));
      }
      ptx::umma_commit(done);
      ptx::umma_commit(drainb);
      ptx::mbar_wait<false>(drainb, 0, 0xffffffffu, kWaitNs);
    }
    __syncwarp();
  }
  if (xcomb && warp >= 2) {
    // merge this group's (head's) split partials into the resident X slice:
    // o_lat[b][c] = sum_s exp(lse_s - m) o_part_s[b][c] / sum_s exp(lse_s - m),
    // with m = max_s lse_s, in the same order and precision as the merge kernel
    const int ct = static_cast<int>(threadIdx.x) - 64;
    const int S = p.comb_splits, H = p.num_heads, h = group;
    float* invz = wts + p.n * S;
    for (int b = ct; b < p.n; b += kCombThreads) {
      float mm = -INFINITY;
      // (unrolled: eight loads in flight rather than one round trip per split)
      if (b < p.batch) {
#pragma unroll 8
        for (int sp = 0; sp < S; ++sp) mm = fmaxf(mm, p.comb_lse[(static_cast<long>(b) * S + sp) * H + h]);
      }
      float z = 0.f;
#pragma unroll 8
      for (int sp = 0; sp < S; ++sp) {
        const float w = (b >= p.batch || mm == -INFINITY) ? 0.f
                                                           : __expf(p.comb_lse[(static_cast<long>(b) * S + sp) * H + h] - mm);
        wts[b * S + sp] = w;
        z += w;
      }
      invz[b] = z > 0.f ? 1.f / z : 0.f;
      if (p.comb_lse_out != nullptr && b < p.batch)
        p.comb_lse_out[static_cast<long>(b) * H + h] = z > 0.f ? mm + __logf(z) : -INFINITY;
    }
    ptx::mbar_arrive(wready);
    const bool wok = wait(wready, 0);
    if (wok) {
      const int d8 = p.d_c / 8;
      const uint4* op = reinterpret_cast<const uint4*>(p.comb_opart);   // 8 fp16 per head and group
      // 16-byte unit u: row b, K chunk k, unit v (columns 64k + 8v .. +7).  A
      // thread takes kU units at a time and loads two splits of all of them
      // before it accumulates, so that 16 loads are in flight, not 1
      constexpr int kU = 8;
      const int total = p.n * 8 * p.x_chunks;
      for (int ub = ct; ub < total; ub += kCombThreads * kU) {
        int bq[kU];
        long base[kU];
        float acc[kU][8];
#pragma unroll
        for (int q = 0; q < kU; ++q) {
          const int u = ub + q * kCombThreads;
          const int b = u / (8 * p.x_chunks), k = (u / 8) % p.x_chunks, v = u % 8;
          bq[q] = u < total ? b : -1;
          base[q] = (static_cast<long>(b) * S * d8 + 8 * k + v) * H + h;
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[q][e] = 0.f;
        }
        for (int sp = 0; sp < S; sp += 2) {
          uint4 x[2][kU];
#pragma unroll
          for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int q = 0; q < kU; ++q)
              if (sp + j < S && bq[q] >= 0 && bq[q] < p.batch)
                x[j][q] = op[base[q] + static_cast<long>(sp + j) * d8 * H];
#pragma unroll
          for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int q = 0; q < kU; ++q)
              if (sp + j < S && bq[q] >= 0 && bq[q] < p.batch) {
                const float w = wts[bq[q] * S + sp + j];
                const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&x[j][q].x));
                const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&x[j][q].y));
                const float2 f2 = __half22float2(*reinterpret_cast<const __half2*>(&x[j][q].z));
                const float2 f3 = __half22float2(*reinterpret_cast<const __half2*>(&x[j][q].w));
                const float4 x0 = make_float4(f0.x, f0.y, f1.x, f1.y), x1 = make_float4(f2.x, f2.y, f3.x, f3.y);
                float* a = acc[q];
                a[0] += w * x0.x; a[1] += w * x0.y; a[2] += w * x0.z; a[3] += w * x0.w;
                a[4] += w * x1.x; a[5] += w * x1.y; a[6] += w * x1.z; a[7] += w * x1.w;
              }
        }
#pragma unroll
        for (int q = 0; q < kU; ++q) {
          const int b = bq[q];
          if (b < 0) continue;
          const int u = ub + q * kCombThreads, k = (u / 8) % p.x_chunks, v = u % 8;
          uint4 pk;
          uint32_t* pw = reinterpret_cast<uint32_t*>(&pk);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const __nv_bfloat162 bb =
                __floats2bfloat162_rn(acc[q][2 * e] * invz[b], acc[q][2 * e + 1] * invz[b]);
            pw[e] = *reinterpret_cast<const uint32_t*>(&bb);
          }
          *reinterpret_cast<uint4*>(smem + k * (p.n * 128) + b * 128 + ((v ^ (b & 7)) << 4)) = pk;
          if (p.comb_olat != nullptr && b < p.batch)
            *reinterpret_cast<uint4*>(p.comb_olat + (static_cast<long>(b) * H + h) * p.d_c + 64 * k + 8 * v) = pk;
        }
      }
    }
    ptx::fence_proxy_async_cta();     // generic writes -> the MMAs' reads of X
    ptx::mbar_arrive(xfull);
  }
  if (warp >= 4) {
    const int q = warp & 3;
    const int m = q * 32 + lane;                       // row of this thread in a tile
    const uint32_t lb = static_cast<uint32_t>(q * 32) << 16;
    if (kEpi == Epi::kAbsorb && mt0 == 0 && split == 0) {
      // RoPE(q_pe[b][h], pos[b]) -> q_lat[b][h][d_c:], pairs (i, i + d_r/2).  Each
      // thread takes up to 8 pairs per round and issues all their loads before
      // any store: the positions in one round trip, then the rotation factors and
      // q_pe values that depend on them in a second (a loop that stores between
      // its loads would pay two round trips per pair).
      constexpr int kPer = 8;
      const int half = p.d_r / 2, total = p.batch * half;
      __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.out);
      for (int base = m; base < total; base += 128 * kPer) {
        int ps[kPer];
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
          const int idx = base + 128 * u;
          ps[u] = idx < total ? __ldg(p.pos + idx / half) : 0;
        }
        float2 r[kPer];
        float x1[kPer], x2[kPer];
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
          const int idx = base + 128 * u;
          const int b = idx / half, i = idx % half;
          const bool ok = idx < total && ps[u] >= 0 && ps[u] < p.max_position;
          r[u] = ok ? __ldg(p.rope_cs + static_cast<long>(ps[u]) * half + i) : make_float2(0.f, 0.f);
          const long qb = (static_cast<long>(b) * p.num_heads + group) * p.d_r;
          x1[u] = ok ? __bfloat162float(p.q_pe[qb + i]) : 0.f;
          x2[u] = ok ? __bfloat162float(p.q_pe[qb + half + i]) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
          const int idx = base + 128 * u;
          if (idx >= total) continue;
          if (ps[u] < 0 || ps[u] >= p.max_position) {
            report_error(p.err, MLA_ERR_BAD_INDEX);
            continue;
          }
          const int b = idx / half, i = idx % half;
          const long ob = b * p.out_ld + group * p.out_group + p.d_c;
          out[ob + i] = __float2bfloat16_rn(x1[u] * r[u].x - x2[u] * r[u].y);
          out[ob + half + i] = __float2bfloat16_rn(x2[u] * r[u].x + x1[u] * r[u].y);
        }
      }
    }
    bool ok = wait(done, 0);
    ok = __all_sync(0xffffffffu, ok);
    if (ok && nst > 0) {
      ptx::tc_fence_after();
      for (int t = 0; t < nacc; ++t) {
        const int m0 = (mt0 + t) * kM;
        for (int c0 = 0; c0 < p.n; c0 += 32) {
          uint32_t v[32];
          ptx::tmem_ld32(tmem + lb + ncpt * t + c0, v);
          ptx::tmem_wait_ld();
          if (kEpi == Epi::kPartialF32) {
            float* out = reinterpret_cast<float*>(p.out) +
                         (sk ? static_cast<long>(blockIdx.x * p.mt_per_cta + t) * p.out_split + m
                             : split * p.out_split + group * p.out_group + m0 + m);
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (c0 + e < p.batch) out[(c0 + e) * p.out_ld] = __uint_as_float(v[e]);
          } else {
            __nv_bfloat16* out =
                reinterpret_cast<__nv_bfloat16*>(p.out) + group * p.out_group + m0 + m;
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (c0 + e < p.batch) out[(c0 + e) * p.out_ld] = __float2bfloat16_rn(__uint_as_float(v[e]));
          }
        }
      }
      ptx::tc_fence_before();
    }
  }
  __syncwarp();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, ncols);
  }
}

// The CTA of a stream-K grid of g CTAs over `units` stages that owns stage u
// (32-bit arithmetic: the launcher keeps units * g below 2^31).
__device__ __forceinline__ int stream_k_owner(int u, int units, int g) {
  int c = u * g / units;
  while (c + 1 < g && (c + 1) * units / g <= u) ++c;
  while (c > 0 && c * units / g > u) --c;
  return c;
}

// y[b][m] = sum over the CTAs c that touched M tile m / 128, in increasing c,
// of partial[c * slots + t][b][m % 128] (t: the tile's place among c's tiles),
// in bf16.  Block (mt, j) covers rows 2j, 2j + 1 of tile mt; its loads are all
// issued before the in-order sum.
constexpr int kReduceMaxParts = 8;
__global__ void __launch_bounds__(256) reduce_stream_k_kernel(const float* __restrict__ part,
                                                              __nv_bfloat16* __restrict__ y, int batch,
                                                              int d_model, int units, int box, int g,
                                                              int slots) {
  grid_dep_wait();
  grid_dep_trigger();
  const int mt = blockIdx.x, r = threadIdx.x & (kM - 1);
  const int b = blockIdx.y * 2 + (threadIdx.x >> 7);
  __shared__ int cs[2];
  if (threadIdx.x == 0) {
    cs[0] = stream_k_owner(mt * box, units, g);
    cs[1] = stream_k_owner((mt + 1) * box - 1, units, g);
  }
  __syncthreads();
  const int c0 = cs[0], c1 = cs[1];
  if (b >= batch) return;
  auto at = [&](int c) {
    const int t = mt - (c * units / g) / box;
    return part[(static_cast<long>(c * slots + t) * batch + b) * kM + r];
  };
  float v[kReduceMaxParts];
#pragma unroll
  for (int k = 0; k < kReduceMaxParts; ++k) v[k] = c0 + k <= c1 ? at(c0 + k) : 0.f;
  float s = 0.f;
#pragma unroll
  for (int k = 0; k < kReduceMaxParts; ++k)
    if (c0 + k <= c1) s += v[k];
  for (int c = c0 + kReduceMaxParts; c <= c1; ++c) s += at(c);
  y[static_cast<long>(b) * d_model + mt * kM + r] = __float2bfloat16_rn(s);
}

// y[b][m] = sum_s partial[s][b][m] in bf16.
__global__ void __launch_bounds__(256) reduce_splits_kernel(const float* __restrict__ part,
                                                            __nv_bfloat16* __restrict__ y,
                                                            int splits, long count) {
  grid_dep_wait();
  grid_dep_trigger();
  for (long i = blockIdx.x * 256L + threadIdx.x; i < count; i += gridDim.x * 256L) {
    float s = 0.f;
    for (int k = 0; k < splits; ++k) s += part[k * count + i];
    y[i] = __float2bfloat16_rn(s);
  }
}

}  // namespace gemm
}  // namespace mla

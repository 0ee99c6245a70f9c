// kvq_encode_tc.cu -- the SRFT-int4 encode on the 5th-generation tensor cores.
//
// The encode of "When Quantization Is Free" (gist.science/de/paper/2605.05699,
// "Methodik" 1-2) is linear up to the quantiser: y = Lambda F_r diag(s) x. For a
// tile of 128 vectors this is a GEMM Y[128 x D] = X[128 x D] W^T with the
// per-plan matrix W = Lambda F_r diag(s), which tcgen05.mma runs with fp32
// accumulators in tensor memory (TMEM). fp16 operands carry W as an exact
// hi + lo pair (W = W_hi + W_lo + O(2^-22 |W|)); x is fp16 already, so both
// products are exact and only the fp32 accumulation rounds.
//
//   [Y_hi | Y_lo] = X [W_hi ; W_lo]^T as one N = 256 product per K step of 16 (the
//   X tile is read once per K step), Y = Y_hi + Y_lo in the epilogue. An MMA has
//   N <= 256, so a CTA produces 128 channels:
//   D = 128: one CTA per tile, all channels, K = 128;
//   D = 256: two CTAs per tile (a CTA pair walks the same tiles), each with one
//            half of the channels and its half of W resident (128 KB), K = 256;
//            the pair's second read of each X tile is served by L2.
//
// Roles (one CTA per SM, persistent over a contiguous range of tiles):
//   warp 0      TMA producer: the plan's W (resident, reloaded when the job
//               changes) and a ring of ten 16 KB K-chunks of X tiles (128-byte
//               swizzle), each freed as soon as the MMAs reading it complete;
//   warp 1      TMEM allocation and the single MMA-issuing thread;
//   warps 2-9   epilogue: one thread per (vector, half of the channel groups);
//               two warps per TMEM lane quarter; 32 columns per tcgen05.ld,
//               group abs-max, fp16 scale, int4 rounding, nibble packing,
//               16-byte code stores and one scale store per half vector.
// Two TMEM accumulators (2 x D columns) let the epilogue of tile i overlap the
// MMAs of tile i + 1. Every wait is bounded; a CTA that gives up raises a device
// error flag and still deallocates its TMEM.
//
// Exact W (EX, plans of the SRHT variant): W = H diag(s) has entries +-1, exact in
// fp16, so one product per K step gives Y exactly up to the fp32 accumulation; the
// per-channel factor lambda_c / sqrt(D) is applied in the epilogue. An MMA then
// covers all D channels (N = D), one CTA per tile at either head dim, half the
// tensor work of the hi/lo product.
#include <algorithm>
#include <cstdio>
#include <mutex>
#include <utility>

#include "kvq_internal.h"
#include "kvq_ptx.cuh"
#include "kvq_quant.cuh"
#include "srft_fft.cuh"

namespace kvq {

__device__ uint32_t g_enc_tc_err = 0;

namespace {

constexpr int kTcRows = 128;    // vectors per tile (MMA M)

constexpr int kTcEpiWarps = 8;  // two per TMEM lane quarter, each taking half the channel groups
constexpr int kTcThreads = 32 * (2 + kTcEpiWarps);
constexpr int kTcMaxJobs = 64;

struct alignas(64) TcJob {
  CUtensorMap xmap;  // x as [rows][D] fp16, box {64, 128}, 128-byte swizzle
  CUtensorMap wmap;  // W as [2D][D] fp16 (hi rows, then lo rows; EX: [D][D]), box {64, N}, 128-byte swizzle
  uint8_t* codes;    // [BH][T_cap][D * BITS / 8]
  uint16_t* scales;  // [BH][T_cap][D/G]
  const float* chan; // EX: the per-channel factors lambda_c / sqrt(D); split: lambda_c dg_c
  const uint32_t* sgn;  // split: sign masks, one per fp16 pair of samples
  int rows, n, T_cap, pos, tile0;  // rows = B*H*n; tile0 = first global tile of the job
};

template <int MAXJ>
struct TcBatch {
  TcJob j[MAXJ];
  int njobs, ntiles;
};

template <int D, bool EX>
struct TcCfg {
  static constexpr int KC = D / 64;                  // 64-wide K chunks (one 128-byte swizzle atom each)
  static constexpr int kSplit = EX ? 1 : D / 128;    // CTAs per tile (channel halves)
  static constexpr int kChunkA = kTcRows * 128;      // one K chunk of a 128-row X tile: 16 KB
  static constexpr int kN = EX ? D : 256;            // MMA N: D exact rows, or 128 W_hi rows then 128 W_lo rows
  static constexpr int kChunkW = kN * 128;           // one K chunk of W
  static constexpr int kW = KC * kChunkW;            // 64 KB (D = 128) or 128 KB (D = 256); EX: 32 / 128 KB
  static constexpr int kChunks = (EX && D == 128) ? 12 : (D == 128 ? 10 : 6);  // X ring depth in K chunks
  static constexpr int kTmemCols = 2 * kN;           // two accumulators of N fp32 columns
  static constexpr int kBars = 8 * (2 * kChunks + 4 + 3) + 16;
  static constexpr int kSmem = kW + kChunks * kChunkA + kBars + 1024;
  static_assert(kSmem <= 227 * 1024, "shared memory");
};

__device__ __forceinline__ int job_of(const TcJob* jobs, int njobs, int job, int t) {
  while (job + 1 < njobs && jobs[job + 1].tile0 <= t) ++job;
  return job;
}

// The quantiser over one 32-channel chunk: one group of 32 or two of 16 (sb: their
// scales); BITS code words (the chunk's 16 or 32 code bytes).
template <int G, int BITS>
__device__ __forceinline__ void quantize_chunk(const float (&y)[32], uint32_t (&w)[BITS], uint32_t (&sb)[32 / G]) {
  if constexpr (G == 32) {
    quantize_group<32, BITS>(y, w, sb[0]);
  } else {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      float yh[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) yh[i] = y[16 * j + i];
      uint32_t wh[BITS / 2];
      quantize_group<16, BITS>(yh, wh, sb[j]);
#pragma unroll
      for (int i = 0; i < BITS / 2; ++i) w[(BITS / 2) * j + i] = wh[i];
    }
  }
}

// the code bytes of 32-channel chunk k of cache row `orow` (16 or 32 bytes)
template <int D, int BITS>
__device__ __forceinline__ void store_chunk(uint8_t* codes, size_t orow, int k, const uint32_t (&w)[BITS]) {
  uint4* row = reinterpret_cast<uint4*>(codes + orow * (D * BITS / 8));
  if constexpr (BITS == 4) {
    row[k] = make_uint4(w[0], w[1], w[2], w[3]);
  } else {
    row[2 * k] = make_uint4(w[0], w[1], w[2], w[3]);
    row[2 * k + 1] = make_uint4(w[4], w[5], w[6], w[7]);
  }
}

// n consecutive fp16 scale bits (n = 2, 4 or 8) to one 4-, 8- or 16-byte store
template <int N>
__device__ __forceinline__ void store_scales(uint16_t* dst, const uint32_t (&sb)[N]) {
  static_assert(N == 2 || N == 4 || N == 8, "scale count");
  if constexpr (N == 2) {
    *reinterpret_cast<uint32_t*>(dst) = sb[0] | (sb[1] << 16);
  } else if constexpr (N == 4) {
    *reinterpret_cast<uint2*>(dst) = make_uint2(sb[0] | (sb[1] << 16), sb[2] | (sb[3] << 16));
  } else {
    *reinterpret_cast<uint4*>(dst) = make_uint4(sb[0] | (sb[1] << 16), sb[2] | (sb[3] << 16), sb[4] | (sb[5] << 16),
                                                sb[6] | (sb[7] << 16));
  }
}

template <int D, bool EX, int G, int BITS, int MAXJ>
__global__ void __launch_bounds__(kTcThreads, 1) encode_tc_kernel(const __grid_constant__ TcBatch<MAXJ> bt) {
  using C = TcCfg<D, EX>;
  constexpr int kTcChunks = C::kChunks;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sW = sm;
  uint8_t* sA = sm + C::kW;
  uint64_t* afull = reinterpret_cast<uint64_t*>(sA + kTcChunks * C::kChunkA);
  uint64_t* aempty = afull + kTcChunks;
  uint64_t* tfull = aempty + kTcChunks;
  uint64_t* tempty = tfull + 2;
  uint64_t* wfull = tempty + 2;
  uint64_t* wempty = wfull + 1;
  uint64_t* mdone = wempty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mdone + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // D = 256: CTAs 2p and 2p + 1 take the same tiles, channel halves 0 and 1
  const int half = C::kSplit == 2 ? (int)(blockIdx.x & 1) : 0;
  const int nwalk = (int)gridDim.x / C::kSplit, walker = (int)blockIdx.x / C::kSplit;
  const int per = (bt.ntiles + nwalk - 1) / nwalk;
  const int t_begin = walker * per;
  const int t_end = min(t_begin + per, bt.ntiles);
  const int ntile = max(0, t_end - t_begin);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kTcChunks; ++s) {
      mbar_init(&afull[s], 1);
      mbar_init(&aempty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], kTcEpiWarps);  // one arrival per epilogue warp
    }
    mbar_init(wfull, 1);
    mbar_init(wempty, 1);
    mbar_init(mdone, 1);
    fence_mbarrier_init();
  }
  // programmatic dependent launch: the next kernel in the stream may start its own
  // prologue now (it reads what this kernel writes only after its grid dependency wait)
  grid_dep_launch();
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && ntile > 0) {
      const uint64_t pol = l2_evict_first_policy();
      int job = job_of(bt.j, bt.njobs, 0, t_begin), wjob = -1, nw = 0;
      // the first job's W (a plan constant, written once when the plan is made) is
      // loaded while the previous kernel in the stream finishes; the inputs after it
      mbar_arrive_expect_tx(wfull, C::kW);
#pragma unroll
      for (int kc = 0; kc < C::KC; ++kc) tma_load_2d(sW + kc * C::kChunkW, &bt.j[job].wmap, wfull, kc * 64, 256 * half);
      wjob = job;
      nw = 1;
      grid_dep_wait();
      for (int i = 0; i < ntile; ++i) {
        const int t = t_begin + i;
        job = job_of(bt.j, bt.njobs, job, t);
        const TcJob& J = bt.j[job];
        if (job != wjob) {
          if (nw > 0 && !mbar_wait_bounded(wempty, (nw - 1) & 1)) {
            atomicOr(&g_enc_tc_err, kErrTimeoutLoad);
            break;
          }
          mbar_arrive_expect_tx(wfull, C::kW);
#pragma unroll
          for (int kc = 0; kc < C::KC; ++kc) tma_load_2d(sW + kc * C::kChunkW, &J.wmap, wfull, kc * 64, 256 * half);
          wjob = job;
          ++nw;
        }
        // the tile's K chunks, each into the next slot of the chunk ring
        const int row = (t - J.tile0) * kTcRows;
        bool ok = true;
#pragma unroll
        for (int kc = 0; kc < C::KC; ++kc) {
          const int c = i * C::KC + kc, s = c % kTcChunks;
          if (c >= kTcChunks && !mbar_wait_bounded(&aempty[s], ((c / kTcChunks) - 1) & 1)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&afull[s], C::kChunkA);
          tma_load_2d_hint(sA + s * C::kChunkA, &J.xmap, &afull[s], kc * 64, row, pol);
        }
        if (!ok) {
          atomicOr(&g_enc_tc_err, kErrTimeoutLoad);
          break;
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && ntile > 0) {
      constexpr uint32_t idesc = umma_idesc_f16(kTcRows, C::kN);
      int job = job_of(bt.j, bt.njobs, 0, t_begin), wjob = -1, nw = 0;
      for (int i = 0; i < ntile; ++i) {
        const int t = t_begin + i;
        job = job_of(bt.j, bt.njobs, job, t);
        if (job != wjob) {
          if (nw > 0) umma_commit(wempty);  // W may be replaced once the MMAs issued so far are done
          if (!mbar_wait_bounded(wfull, nw & 1)) {
            atomicOr(&g_enc_tc_err, kErrTimeoutLoad);
            break;
          }
          wjob = job;
          ++nw;
        }
        const int a = i & 1;
        if (i >= 2 && !mbar_wait_bounded(&tempty[a], ((i >> 1) - 1) & 1)) {
          atomicOr(&g_enc_tc_err, kErrTimeoutLoad);
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(a * C::kN);
        const uint32_t w0 = smem_u32(sW);
        bool ok = true;
#pragma unroll
        for (int kc = 0; kc < C::KC; ++kc) {
          const int c = i * C::KC + kc, s = c % kTcChunks;
          if (!mbar_wait_bounded(&afull[s], (c / kTcChunks) & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + s * C::kChunkA);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {  // K = 16 per MMA: 32 bytes along the swizzled row
            const uint64_t ad = umma_desc_sw128(a0 + kk * 32);
            const uint64_t wd = umma_desc_sw128(w0 + kc * C::kChunkW + kk * 32);
            umma_f16(d, ad, wd, idesc, (kc | kk) != 0);
          }
          umma_commit(&aempty[s]);  // this chunk is free once these MMAs have read it
        }
        if (!ok) {
          atomicOr(&g_enc_tc_err, kErrTimeoutLoad);
          break;
        }
        umma_commit(&tfull[a]);  // the accumulator is ready for the epilogue
      }
      // TMEM is released below: wait (bounded) until every MMA of this CTA has completed
      // (a commit with nothing outstanding arrives at once)
      umma_commit(mdone);
      if (!mbar_wait_bounded(mdone, 0)) atomicOr(&g_enc_tc_err, kErrTimeoutLoad);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // warp w: TMEM lanes 32 (w % 4) .. + 31 (one vector per thread), channel groups
    // [h * NGH, (h + 1) * NGH) of the CTA's channels with h = (w - 2) / 4
    constexpr int NGH = EX ? D / 64 : 2;  // 32-channel chunks per thread: two threads per vector
    constexpr int SPC = 32 / G;            // scale groups per chunk
    const int q = warp & 3;
    const int h = (warp - 2) >> 2;
    int job = ntile > 0 ? job_of(bt.j, bt.njobs, 0, t_begin) : 0;
    for (int i = 0; i < ntile; ++i) {
      const int t = t_begin + i;
      job = job_of(bt.j, bt.njobs, job, t);
      const TcJob& J = bt.j[job];
      const int a = i & 1;
      // warp-uniform outcome: the tcgen05.ld below needs the whole warp
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(&tfull[a], (i >> 1) & 1))) {
        if (lane == 0) atomicOr(&g_enc_tc_err, kErrTimeoutLoad);
        break;
      }
      tc_fence_after();
      const int r = (t - J.tile0) * kTcRows + 32 * q + lane;  // row of this thread's vector in the job
      const bool valid = r < J.rows;
      const int bh = valid ? r / J.n : 0;
      const size_t orow = (size_t)bh * J.T_cap + J.pos + (r - bh * J.n);
      const uint32_t ta = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(a * C::kN + 32 * NGH * h);
      uint32_t sb[NGH * SPC];
      if constexpr (EX) {
        // Y exact up to the fp32 accumulation; y = Y * lambda_c / sqrt(D)
        float y[NGH][32];
#pragma unroll
        for (int g = 0; g < NGH; ++g) tmem_ld32(ta + 32 * g, y[g]);
        tmem_ld_wait();
#pragma unroll
        for (int g = 0; g < NGH; ++g) tmem_regs_fence(y[g]);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[a]);
#pragma unroll
        for (int g = 0; g < NGH; ++g) {
          const float4* f4 = reinterpret_cast<const float4*>(J.chan + 32 * (NGH * h + g));
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float4 f = __ldg(f4 + e);
            y[g][4 * e] *= f.x;
            y[g][4 * e + 1] *= f.y;
            y[g][4 * e + 2] *= f.z;
            y[g][4 * e + 3] *= f.w;
          }
          uint32_t w[BITS], sg[SPC];
          quantize_chunk<G, BITS>(y[g], w, sg);
#pragma unroll
          for (int j = 0; j < SPC; ++j) sb[SPC * g + j] = sg[j];
          if (valid) store_chunk<D, BITS>(J.codes, orow, NGH * h + g, w);
        }
        if (valid) store_scales<NGH * SPC>(J.scales + orow * (D / G) + NGH * SPC * h, sb);
      } else {
        float y[NGH][32], ylo[NGH][32];
#pragma unroll
        for (int g = 0; g < NGH; ++g) {
          tmem_ld32(ta + 32 * g, y[g]);
          tmem_ld32(ta + 128 + 32 * g, ylo[g]);
        }
        tmem_ld_wait();
#pragma unroll
        for (int g = 0; g < NGH; ++g) {
          tmem_regs_fence(y[g]);
          tmem_regs_fence(ylo[g]);
        }
        // the accumulator may be overwritten as soon as every epilogue warp has its values
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[a]);
#pragma unroll
        for (int g = 0; g < NGH; ++g) {
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const float2 v = __fadd2_rn(make_float2(y[g][e], y[g][e + 1]), make_float2(ylo[g][e], ylo[g][e + 1]));
            y[g][e] = v.x;
            y[g][e + 1] = v.y;
          }
          uint32_t w[BITS], sg[SPC];
          quantize_chunk<G, BITS>(y[g], w, sg);
#pragma unroll
          for (int j = 0; j < SPC; ++j) sb[SPC * g + j] = sg[j];
          if (valid) store_chunk<D, BITS>(J.codes, orow, 4 * half + NGH * h + g, w);
        }
        if (valid) store_scales<NGH * SPC>(J.scales + orow * (D / G) + SPC * (4 * half + NGH * h), sb);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}


// ============================================================================ D = 256, radix-2 split
// The SRFT at D = 256 by one radix-2 decimation in time, with the two half-length
// transforms on the tensor cores (half the tensor work of the dense hi/lo product).
// With x' = s (.) x and the unnormalised 128-point real spectra (slot order: slot 0 =
// X_0, slot 1 = X_64, slot 2k = Re X_k, slot 2k+1 = Im X_k)
//   E = F128 x'_even,  O = F128 x'_odd,
//   X_k = E_k + W^k O_k,  X_{128-k} = conj(E_k - W^k O_k),  W = e^{-2 pi i / 256},
// and y_c = lambda_c dg_c (Re or Im of X at channel c's frequency). F128 is the plan-
// independent matrix the attention kernels use (fp16 hi + lo, exact to ~2^-22), so
// it is loaded once per CTA and never reloaded when the job changes; each plan's
// signs are applied while the samples are separated, and its factors in the epilogue.
//   warp 0      TMA: F128 (resident), each tile's plan constants (bulk copies into one
//               of three slots), a ring of 16 KB chunks (128 rows x 64 samples) of x;
//   warp 1      TMEM (E and O of two tiles: 512 columns) and the MMA thread: per tile
//               2 x 2 x 4 K steps of M = 128, N = 128 (hi, then lo into the same
//               accumulator);
//   warps 2-9   workers, per tile i: first the separation of tile i + 1 -- thread
//               (row r, half j) applies the signs to row r of chunk pair j (samples
//               128j .. 128j + 127) and rewrites it in place as the 64 even samples
//               (chunk 2j: E's inputs 64j .. 64j + 63) and the 64 odd ones, so the MMAs
//               of tile i + 1 run during the epilogue of tile i; then the epilogue of
//               tile i -- thread (row, h) forms X_k and X_{128-k} for k = 16 g .. 16 g + 16
//               of its group pairs g = 2h, 2h + 1 (channel chunks g and 7 - g) with
//               compile-time twiddles, applies the factors and quantises.
constexpr int kSpRing = 9;     // ring depth in chunks (a tile is four)
constexpr int kSpWork = 8;     // worker warps: the separation of tile i + 1, then the epilogue of tile i
constexpr int kSpThreads = 32 * (2 + kSpWork);
constexpr int kSpChunk = kTcRows * 128;        // 16 KB
constexpr int kSpF = 2 * (256 * 128);          // F128 [hi; lo] (256 rows) x 2 K-chunks of 64: 64 KB
constexpr int kSpCst = 256 * 4 + 128 * 4;      // a tile's plan constants: lambda_c dg_c [256], sign masks [128]
// constant slots: tiles i (epilogue) and i + 1 (separation) are in use while tile i + 2's
// constants load, so that load never waits for the epilogue just finishing
constexpr int kSpCstSlots = 3;
constexpr int kSpBars = 8 * (3 * kSpRing + 2 * 2 + 2 * kSpCstSlots + 2) + 16;
constexpr int kSpSmem = kSpF + kSpRing * kSpChunk + kSpCstSlots * kSpCst + kSpBars + 1024;
static_assert(kSpSmem <= 227 * 1024, "shared memory");

// 16 bytes of shared memory, loaded where written (volatile: loop-invariant loads of the
// sign masks would otherwise be hoisted out of the row loop and held in 128 registers)
__device__ __forceinline__ uint4 lds128_here(const void* p) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(smem_u32(p)));
  return v;
}

// byte offset of 16-byte unit u of row r in a 128-byte-swizzled chunk (1024-byte aligned)
__device__ __forceinline__ uint32_t sw128_off(int r, int u) { return (uint32_t)(r * 128 + ((u ^ (r & 7)) << 4)); }

// (cos, sin)(2 pi k / 256) for k = 16 GP + TT, at [17 GP + TT] (GP = 0..3, TT = 0..16);
// written once per device from the same exact-octant Taylor evaluation as the
// compile-time twiddles of the register FFT
__constant__ float2 c_split_tw[4 * 17];

// Frequency k = 16 GP + TT of a group pair: X_k = E_k + W^k O_k into chunk GP (y0) and
// X_{128-k} = conj(E_k - W^k O_k) into chunk 7 - GP (y1), W = e^{-2 pi i / 256}, each value
// times its channel factor. GP is a runtime value (one code path for every pair).
template <int TT>
__device__ __forceinline__ void split_freq(int GP, const float (&e)[32], const float (&o)[32], float e32, float e33,
                                           float o32, float o33, const float* c0, const float* c1, float (&y0)[32],
                                           float (&y1)[32]) {
  float er, ei, orr, oi;
  if constexpr (TT == 0) {
    // k = 0: slot 1 holds X_64, and Im X_0 = 0
    er = e[0];
    orr = o[0];
    ei = GP == 0 ? 0.0f : e[1];
    oi = GP == 0 ? 0.0f : o[1];
  } else if constexpr (TT < 16) {
    er = e[2 * TT];
    ei = e[2 * TT + 1];
    orr = o[2 * TT];
    oi = o[2 * TT + 1];
  } else {
    // k = 16 GP + 16: slots (2k, 2k + 1), or for GP = 3 the real E_64 and O_64 (slot 1)
    const bool ny = GP == 3;
    er = ny ? e33 : e32;
    ei = ny ? 0.0f : e33;
    orr = ny ? o33 : o32;
    oi = ny ? 0.0f : o33;
  }
  const float2 w = c_split_tw[17 * GP + TT];
  const float xr = fmaf(w.x, orr, fmaf(w.y, oi, er));   // Re X_k = Re (E + W^k O)
  const float xi = fmaf(w.x, oi, fmaf(-w.y, orr, ei));  // Im X_k
  // chunk GP: channel 2k - 1 = Re X_k (local 2TT - 1), 2k = Im X_k (local 2TT); local 0 of chunk 0 is X_0
  if constexpr (TT >= 1) y0[2 * TT - 1] = xr * c0[2 * TT - 1];
  if constexpr (TT == 0) y0[0] = (GP == 0 ? xr : xi) * c0[0];
  else if constexpr (TT <= 15) y0[2 * TT] = xi * c0[2 * TT];
  // chunk 7 - GP: Re X_{128-k} = 2 Re E - Re X_k at local 31 - 2TT, Im X_{128-k} = Im X_k - 2 Im E at 32 - 2TT
  if constexpr (TT <= 15) y1[31 - 2 * TT] = fmaf(2.0f, er, -xr) * c1[31 - 2 * TT];
  if constexpr (TT >= 1) y1[32 - 2 * TT] = fmaf(-2.0f, ei, xi) * c1[32 - 2 * TT];
}

template <int... TT>
__device__ __forceinline__ void split_freqs(std::integer_sequence<int, TT...>, int GP, const float (&e)[32],
                                            const float (&o)[32], float e32, float e33, float o32, float o33,
                                            const float* c0, const float* c1, float (&y0)[32], float (&y1)[32]) {
  (split_freq<TT>(GP, e, o, e32, e33, o32, o33, c0, c1, y0, y1), ...);
}

// Quantise and store one channel chunk of a tile row (codes and scale bits).
template <int G, int BITS>
__device__ __forceinline__ void split_store(const float (&y)[32], int chunk, uint8_t* codes, uint16_t* srow,
                                            bool valid) {
  constexpr int SPC = 32 / G;
  uint32_t w[BITS], sg[SPC];
  quantize_chunk<G, BITS>(y, w, sg);
  if (valid) {
    store_chunk<256, BITS>(codes, 0, chunk, w);
    if constexpr (SPC == 1) srow[chunk] = (uint16_t)sg[0];
    else *reinterpret_cast<uint32_t*>(srow + 2 * chunk) = sg[0] | (sg[1] << 16);
  }
}

// E_k and O_k (k = 16 GP + tt, tt = 0..16) of one tile row, issued as TMEM loads (the
// caller waits with tmem_ld_wait before using them)
struct SplitIn {
  float e[32], o[32], e32, e33, o32, o33;
};
__device__ __forceinline__ void split_load(SplitIn& v, int GP, uint32_t ta) {
  tmem_ld32(ta + 32 * GP, v.e);
  tmem_ld32(ta + 128 + 32 * GP, v.o);
  // k = 16 GP + 16: slots (2k, 2k + 1), or for GP = 3 the real X_64 in slot 1 (read with slot 0)
  const uint32_t xc = GP < 3 ? 32 * GP + 32 : 0;
  tmem_ld2(ta + xc, v.e32, v.e33);
  tmem_ld2(ta + 128 + xc, v.o32, v.o33);
}
__device__ __forceinline__ void split_fence(SplitIn& v) {
  tmem_regs_fence(v.e);
  tmem_regs_fence(v.o);
  tmem_regs_fence(v.e32);
  tmem_regs_fence(v.e33);
  tmem_regs_fence(v.o32);
  tmem_regs_fence(v.o33);
}

// Group pair GP of a tile row: channel chunks GP (from X_k, k = 16 GP + tt, tt = 0..16) and
// 7 - GP (from X_{128-k}), both formed from one TMEM load of E_k and O_k.
template <int G, int BITS>
__device__ __forceinline__ void split_pair(int GP, uint32_t ta, const float* chan, uint8_t* codes, uint16_t* srow,
                                           bool valid, uint64_t* tempty, bool release) {
  SplitIn v;
  split_load(v, GP, ta);
  tmem_ld_wait();
  split_fence(v);
  if (release) {  // every TMEM value of this tile is in registers: the accumulator may be reused
    tc_fence_before();
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(tempty);
  }
  float y0[32], y1[32];
  split_freqs(std::make_integer_sequence<int, 17>{}, GP, v.e, v.o, v.e32, v.e33, v.o32, v.o33, chan + 32 * GP,
              chan + 32 * (7 - GP), y0, y1);
  split_store<G, BITS>(y0, GP, codes, srow, valid);
  split_store<G, BITS>(y1, 7 - GP, codes, srow, valid);
}

template <int G, int BITS, int MAXJ>
__global__ void __launch_bounds__(kSpThreads, 1) encode_split_kernel(const __grid_constant__ TcBatch<MAXJ> bt) {
  constexpr int SPC = 32 / G;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sF = sm;
  uint8_t* sR = sF + kSpF;
  uint8_t* sC = sR + kSpRing * kSpChunk;
  uint64_t* rfull = reinterpret_cast<uint64_t*>(sC + kSpCstSlots * kSpCst);  // [ring] a chunk landed
  uint64_t* rdone = rfull + kSpRing;                                // [ring] a chunk separated
  uint64_t* rempty = rdone + kSpRing;                               // [ring] the MMAs read it
  uint64_t* tfull = rempty + kSpRing;  // [2] accumulators ready
  uint64_t* tempty = tfull + 2;        // [2] accumulators drained
  uint64_t* cfull = tempty + 2;                // [slots] a tile's plan constants landed
  uint64_t* cempty = cfull + kSpCstSlots;      // [slots] the workers are done with them
  uint64_t* ffull = cempty + kSpCstSlots;      // F128 landed
  uint64_t* mdone = ffull + 1;         // every MMA of this CTA completed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mdone + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int per = (bt.ntiles + (int)gridDim.x - 1) / (int)gridDim.x;
  const int t_begin = (int)blockIdx.x * per;
  const int t_end = min(t_begin + per, bt.ntiles);
  const int ntile = max(0, t_end - t_begin);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSpRing; ++s) {
      mbar_init(&rfull[s], 1);
      mbar_init(&rdone[s], kSpWork / 2);  // the four worker warps of that chunk pair
      mbar_init(&rempty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], kSpWork);
    }
    for (int b = 0; b < kSpCstSlots; ++b) {
      mbar_init(&cfull[b], 1);
      mbar_init(&cempty[b], kSpWork);
    }
    mbar_init(ffull, 1);
    mbar_init(mdone, 1);
    fence_mbarrier_init();
  }
  grid_dep_launch();
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && ntile > 0) {
      const uint64_t pol = l2_evict_first_policy();
      int job = job_of(bt.j, bt.njobs, 0, t_begin);
      // F128 is a constant of every plan (written when the plan is made): loaded while
      // the previous kernel in the stream finishes; the inputs only after it
      mbar_arrive_expect_tx(ffull, kSpF);
      tma_load_2d(sF, &bt.j[job].wmap, ffull, 0, 0);
      tma_load_2d(sF + kSpF / 2, &bt.j[job].wmap, ffull, 64, 0);
      grid_dep_wait();
      bool ok = true;
      for (int i = 0; i < ntile && ok; ++i) {
        const int t = t_begin + i;
        job = job_of(bt.j, bt.njobs, job, t);
        const TcJob& J = bt.j[job];
        const int row = (t - J.tile0) * kTcRows;
        const int cs = i % kSpCstSlots;
        if (i >= kSpCstSlots && !mbar_wait_bounded(&cempty[cs], ((i / kSpCstSlots) - 1) & 1)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&cfull[cs], kSpCst);
        bulk_load(sC + cs * kSpCst, J.chan, 256 * 4, &cfull[cs]);
        bulk_load(sC + cs * kSpCst + 256 * 4, J.sgn, 128 * 4, &cfull[cs]);
#pragma unroll
        for (int kc = 0; kc < 4; ++kc) {
          const int c = 4 * i + kc, s = c % kSpRing;
          if (c >= kSpRing && !mbar_wait_bounded(&rempty[s], ((c / kSpRing) - 1) & 1)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&rfull[s], kSpChunk);
          tma_load_2d_hint(sR + s * kSpChunk, &J.xmap, &rfull[s], kc * 64, row, pol);
        }
      }
      if (!ok) atomicOr(&g_enc_tc_err, kErrTimeoutLoad);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && ntile > 0) {
      constexpr uint32_t idesc = umma_idesc_f16(kTcRows, 128);
      bool ok = mbar_wait_bounded(ffull, 0);
      for (int i = 0; i < ntile && ok; ++i) {
        const int a = i & 1;
        if (i >= 2 && !mbar_wait_bounded(&tempty[a], ((i >> 1) - 1) & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t f0 = smem_u32(sF);
#pragma unroll
        for (int j = 0; j < 2 && ok; ++j) {
#pragma unroll
          for (int eo = 0; eo < 2; ++eo) {  // E's inputs 64j .. 64j + 63 in chunk 4i + 2j, O's in the next
            const int c = 4 * i + 2 * j + eo, s = c % kSpRing;
            if (!mbar_wait_bounded(&rdone[s], (c / kSpRing) & 1)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t d = tmem + (uint32_t)(a * 256 + eo * 128);
            const uint32_t a0 = smem_u32(sR + s * kSpChunk);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {  // K = 16 per MMA: 32 bytes along the swizzled row
              const uint64_t ad = umma_desc_sw128(a0 + kk * 32);
              const uint32_t fb = f0 + j * (kSpF / 2) + kk * 32;
              umma_f16(d, ad, umma_desc_sw128(fb), idesc, (j | kk) != 0);        // F128 hi rows
              umma_f16(d, ad, umma_desc_sw128(fb + 128 * 128), idesc, true);    // F128 lo rows
            }
            umma_commit(&rempty[s]);  // the chunk is free once these MMAs have read it
          }
        }
        if (!ok) break;
        umma_commit(&tfull[a]);
      }
      if (!ok) atomicOr(&g_enc_tc_err, kErrTimeoutLoad);
      // TMEM is released below: wait (bounded) until every MMA of this CTA has completed
      umma_commit(mdone);
      if (!mbar_wait_bounded(mdone, 0)) atomicOr(&g_enc_tc_err, kErrTimeoutLoad);
    }
  } else {
    // ------------------------------------------------------------ workers
    const int wi = warp - 2;
    const int q = warp & 3;        // TMEM lane quarter of this warp (epilogue)
    const int h = wi >> 2;         // epilogue: group pairs 2h and 2h + 1; separation: chunk pair h
    const int srow = 32 * (wi & 3) + lane;  // separation: the row this thread rewrites
    // signs + even/odd separation of row srow of chunk pair h of tile i, in place
    auto separate = [&](int i) -> bool {
      const int cs = i % kSpCstSlots;
      if (!mbar_wait_bounded(&cfull[cs], (i / kSpCstSlots) & 1)) return false;
      const uint4* sg4 = reinterpret_cast<const uint4*>(sC + cs * kSpCst + 256 * 4);  // 8 samples per uint4
      const int c0 = 4 * i + 2 * h;  // chunks c0 (samples 128h .. +63) and c0 + 1 (128h + 64 .. +127)
      const int s0 = c0 % kSpRing, s1 = (c0 + 1) % kSpRing;
      if (!(mbar_wait_bounded(&rfull[s0], (c0 / kSpRing) & 1) && mbar_wait_bounded(&rfull[s1], ((c0 + 1) / kSpRing) & 1)))
        return false;
      uint8_t* p0 = sR + s0 * kSpChunk;
      uint8_t* p1 = sR + s1 * kSpChunk;
      uint4 in[16];  // this row's 128 samples, signs applied
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        uint4 v = *reinterpret_cast<const uint4*>((u < 8 ? p0 : p1) + sw128_off(srow, u & 7));
        const uint4 m = sg4[16 * h + u];
        v.x ^= m.x;
        v.y ^= m.y;
        v.z ^= m.z;
        v.w ^= m.w;
        in[u] = v;
      }
#pragma unroll
      for (int v = 0; v < 8; ++v) {  // unit v: samples 128h + 16v .. + 15 -> 8 even, 8 odd
        const uint4 A = in[2 * v], B = in[2 * v + 1];
        *reinterpret_cast<uint4*>(p0 + sw128_off(srow, v)) =
            make_uint4(prmt(A.x, A.y, 0x5410u), prmt(A.z, A.w, 0x5410u), prmt(B.x, B.y, 0x5410u),
                       prmt(B.z, B.w, 0x5410u));
        *reinterpret_cast<uint4*>(p1 + sw128_off(srow, v)) =
            make_uint4(prmt(A.x, A.y, 0x7632u), prmt(A.z, A.w, 0x7632u), prmt(B.x, B.y, 0x7632u),
                       prmt(B.z, B.w, 0x7632u));
      }
      fence_proxy_async_smem();  // generic-proxy writes -> visible to the tensor cores
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&rdone[s0]);
        mbar_arrive(&rdone[s1]);
      }
      return true;
    };
    bool ok = ntile > 0 ? __all_sync(0xffffffffu, separate(0)) : true;
    int job = ntile > 0 ? job_of(bt.j, bt.njobs, 0, t_begin) : 0;
    for (int i = 0; i < ntile && ok; ++i) {
      if (i + 1 < ntile && !__all_sync(0xffffffffu, separate(i + 1))) {
        ok = false;
        break;
      }
      const int t = t_begin + i;
      job = job_of(bt.j, bt.njobs, job, t);
      const TcJob& J = bt.j[job];
      const int a = i & 1;
      // warp-uniform outcome: the tcgen05.ld below needs the whole warp
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(&tfull[a], (i >> 1) & 1))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int r = (t - J.tile0) * kTcRows + 32 * q + lane;
      const bool valid = r < J.rows;
      const int bh = valid ? r / J.n : 0;
      const size_t orow = (size_t)bh * J.T_cap + J.pos + (r - bh * J.n);
      const uint32_t ta = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(a * 256);
      const float* chan = reinterpret_cast<const float*>(sC + (i % kSpCstSlots) * kSpCst);
      uint8_t* crow = J.codes + orow * (256 * BITS / 8);
      uint16_t* srow = J.scales + orow * (256 / G);
      // group pairs 2h and 2h + 1 in turn (one code path: the i-cache holds the whole loop)
#pragma unroll 1
      for (int pp = 0; pp < 2; ++pp)
        split_pair<G, BITS>(2 * h + pp, ta, chan, crow, srow, valid, &tempty[a], pp == 1);
      __syncwarp();
      if (lane == 0) mbar_arrive(&cempty[i % kSpCstSlots]);
    }
    if (!ok && lane == 0) atomicOr(&g_enc_tc_err, kErrTimeoutLoad);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}


// the split kernel's twiddle table, once per device (the set-up of its first launch there)
kvq_status split_twiddles() {
  static std::mutex mu;
  static bool done[64] = {false};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return fail(KVQ_ERR_DEVICE, "encode: no device");
  std::lock_guard<std::mutex> lk(mu);
  if (!done[dev]) {
    float2 tw[4 * 17];
    for (int gp = 0; gp < 4; ++gp)
      for (int tt = 0; tt <= 16; ++tt)
        tw[17 * gp + tt] = make_float2(static_cast<float>(cos2pi_frac(16 * gp + tt, 256)),
                                       static_cast<float>(sin2pi_frac(16 * gp + tt, 256)));
    if (cudaMemcpyToSymbol(c_split_tw, tw, sizeof(tw)) != cudaSuccess)
      return fail(KVQ_ERR_CUDA, "encode: twiddle table upload failed");
    done[dev] = true;
  }
  return KVQ_OK;
}

void tc_prepare() {
  static std::once_flag once;
  std::call_once(once, [] {
    for (int bits : {4, 8})
      for (int D : {128, 256})
        for (int G : {32, 16})
          dispatch_dgb(D, G, bits, [](auto d, auto g, auto b) {
            constexpr int kD = decltype(d)::value, kG = decltype(g)::value, kB = decltype(b)::value;
            cudaFuncSetAttribute(encode_tc_kernel<kD, false, kG, kB, kTcMaxJobs>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, TcCfg<kD, false>::kSmem);
            cudaFuncSetAttribute(encode_tc_kernel<kD, true, kG, kB, kTcMaxJobs>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, TcCfg<kD, true>::kSmem);
            if constexpr (kD == 256)
              cudaFuncSetAttribute(encode_split_kernel<kG, kB, kTcMaxJobs>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, kSpSmem);
            return 0;
          });
  });
}

template <int D, bool EX, int G, int BITS>
cudaError_t tc_launch(cudaLaunchConfig_t cfg, const TcBatch<kTcMaxJobs>& bt, int tiles, int sms) {
  cfg.gridDim = dim3(TcCfg<D, EX>::kSplit == 2 ? 2 * std::min(tiles, sms / 2) : std::min(tiles, sms));
  cfg.dynamicSmemBytes = TcCfg<D, EX>::kSmem;
  return cudaLaunchKernelEx(&cfg, encode_tc_kernel<D, EX, G, BITS, kTcMaxJobs>, bt);
}

template <int G, int BITS>
cudaError_t split_launch(cudaLaunchConfig_t cfg, const TcBatch<kTcMaxJobs>& bt, int tiles, int sms) {
  cfg.gridDim = dim3(std::min(tiles, sms));
  cfg.blockDim = dim3(kSpThreads);
  cfg.dynamicSmemBytes = kSpSmem;
  return cudaLaunchKernelEx(&cfg, encode_split_kernel<G, BITS, kTcMaxJobs>, bt);
}

}  // namespace

bool encode_tc_supported(int D, int G) { return (D == 128 || D == 256) && (G == 32 || G == 16); }

bool encode_split_supported(const kvq_plan* p) { return p->D == 256 && p->xform == 0 && (p->G == 32 || p->G == 16); }

// Grouped launch over jobs of one head_dim (128 or 256), group (32 or 16), transform and
// code width (4 or 8 bits); jobs with no rows are skipped. split: the radix-2 split
// kernel (D = 256, SRFT plans) instead of the dense product.
kvq_status launch_encode_tc(const kvq_encode_job* jobs, int njobs, cudaStream_t strm, bool split) {
  const int D = jobs[0].plan->D;
  const bool ex = jobs[0].plan->xform == 1;  // SRHT: exact W
  if (split && !encode_split_supported(jobs[0].plan))
    return fail(KVQ_ERR_UNSUPPORTED, "encode: the radix-2 split kernel serves head_dim 256 SRFT plans");
  tc_prepare();
  if (split) {
    const kvq_status st = split_twiddles();
    if (st != KVQ_OK) return st;
  }
  int i0 = 0;
  while (i0 < njobs) {
    TcBatch<kTcMaxJobs> bt{};
    int nj = 0, tiles = 0;
    int i = i0;
    for (; i < njobs && nj < kTcMaxJobs; ++i) {
      const kvq_encode_job& j = jobs[i];
      const long rows = (long)j.B * j.H * j.n;
      if (rows == 0) continue;
      if (rows > (1l << 31) - 1) return fail(KVQ_ERR_UNSUPPORTED, "encode: more than 2^31 - 1 vectors in one job");
      TcJob& J = bt.j[nj];
      const uint64_t xd[2] = {(uint64_t)D, (uint64_t)rows};
      const uint64_t xs[1] = {(uint64_t)D * 2};
      const uint32_t xb[2] = {64u, (uint32_t)kTcRows};
      kvq_status st = encode_tiled(&J.xmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, j.x, xd, xs, xb,
                                   CU_TENSOR_MAP_SWIZZLE_128B, "encode x");
      if (st != KVQ_OK) return st;
      // W = Lambda F_r diag(s): per 128-channel half, 128 hi rows then 128 lo rows, D
      // columns; exact W (SRHT): H diag(s), D rows (channels), D columns
      // split: F128 [hi 128 rows; lo 128 rows] x 128 columns (the plan-independent operand)
      if (split) {
        const uint64_t fd[2] = {128u, 256u};
        const uint64_t fs[1] = {256u};
        const uint32_t fb[2] = {64u, 256u};
        st = encode_tiled(&J.wmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, j.plan->rot_dev, fd, fs, fb,
                          CU_TENSOR_MAP_SWIZZLE_128B, "encode F128");
      } else {
        const uint64_t wd[2] = {(uint64_t)D, (uint64_t)(ex ? D : 2 * D)};
        const uint64_t ws[1] = {(uint64_t)D * 2};
        const uint32_t wb[2] = {64u, (uint32_t)(ex ? D : 256)};
        st = encode_tiled(&J.wmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, j.plan->wt_dev, wd, ws, wb,
                          CU_TENSOR_MAP_SWIZZLE_128B, "encode weights");
      }
      if (st != KVQ_OK) return st;
      J.codes = j.codes;
      J.scales = j.scales;
      J.chan = j.plan->enc_dev->chan;
      J.sgn = j.plan->enc_dev->sgn;
      J.rows = (int)rows;
      J.n = j.n;
      J.T_cap = j.T_cap;
      J.pos = j.pos;
      J.tile0 = tiles;
      tiles += (int)((rows + kTcRows - 1) / kTcRows);
      ++nj;
    }
    i0 = i;
    if (nj == 0) continue;
    bt.njobs = nj;
    bt.ntiles = tiles;
    int dev = 0;
    cudaGetDevice(&dev);
    const int sms = num_sms(dev);
    // programmatic dependent launch: the kernel loads its first W and allocates TMEM
    // while the previous kernel in the stream finishes (grid dependency wait before the
    // inputs and every global write)
    cudaLaunchConfig_t cfg{};
    cfg.blockDim = dim3(kTcThreads);
    cfg.stream = strm;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = dispatch_dgb(D, jobs[0].plan->G, jobs[0].plan->bits, [&](auto d, auto g, auto b) {
      constexpr int kD = decltype(d)::value, kG = decltype(g)::value, kB = decltype(b)::value;
      if (split) return split_launch<kG, kB>(cfg, bt, tiles, sms);
      return ex ? tc_launch<kD, true, kG, kB>(cfg, bt, tiles, sms) : tc_launch<kD, false, kG, kB>(cfg, bt, tiles, sms);
    });
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return fail(KVQ_ERR_CUDA, std::string("encode (tensor cores) launch: ") + cudaGetErrorString(e));
  }
  return KVQ_OK;
}

uint32_t encode_tc_error_flags(bool clear) {
  uint32_t v = 0;
  cudaMemcpyFromSymbol(&v, g_enc_tc_err, sizeof(v));
  if (clear && v) {
    const uint32_t z = 0;
    cudaMemcpyToSymbol(g_enc_tc_err, &z, sizeof(z));
  }
  return v;
}

}  // namespace kvq

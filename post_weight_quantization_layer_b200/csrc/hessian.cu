// Calibration Hessian accumulation H += 2 X^T X on the 5th-generation tensor cores.
//
// Source: "第5章 GPTQ 实战" §5.1.7 — the reconstruction error ||(W - W_q) X||^2 is a
// quadratic form whose Hessian is X X^T up to a constant (here 2), estimated from the
// calibration activations.  With X stored tokens x channels the product is X^T X: a
// SYRK whose contraction runs over tokens.
//
// Design (sm_100a):
// * Output tiles of 128 (rows i) x 256 (cols j) of H; only tiles touching the upper
//   triangle are computed and each element is added to both H[i][j] and H[j][i].
// * Persistent grid, one CTA per SM, walking (tile, token segment) units in the order of
//   hessian_sched.cuh: each wave of CTAs works on one token segment of a compact group of
//   tiles, so the CTAs stream the same token rows in step and each row of X is fetched
//   from DRAM a few times instead of once per tile; a CTA's consecutive units of one
//   tile accumulate without write-back, and its epilogue overlaps its next unit's MMAs.
// * A warp-specialised CTA of 10 warps: warp 0 issues TMA loads of X (channels
//   contiguous, 128-byte swizzle) into a 4-stage shared-memory ring; warp 1 issues
//   tcgen05.mma kind::f16 (A and B both MN-major, since X^T and X come from the
//   same row-major X) into a TMEM accumulator; warps 2..9 drain the accumulator.
// * The tensor-core accumulator is drained every FLUSH_KSTEPS*64 tokens into fp32
//   registers (two TMEM buffers of 256 columns, ping-pong), so a long token range
//   never rides on one hardware accumulator; the CTA's total is added to H with
//   fp32 atomics at the end.
#include <cuda.h>

#include <algorithm>
#include <atomic>
#include <mutex>

#include "common.cuh"
#include "hessian_sched.cuh"
#include "sm100.cuh"

namespace gptq {
namespace {

using namespace sm100;

constexpr int BM = 128;          // rows (i) per tile = UMMA M
constexpr int BN = 256;          // cols (j) per tile = UMMA N
constexpr int BK = 64;           // tokens per pipeline stage
constexpr int STAGES = 4;
constexpr int BOX_BYTES = 64 * BK * 2;             // one TMA box: 64 channels x 64 tokens x 2 B
constexpr int A_BYTES = BM * BK * 2;               // 2 boxes
constexpr int B_BYTES = BN * BK * 2;               // 4 boxes
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;     // 48 KiB
constexpr int FLUSH_KSTEPS = 16;                   // drain every 1024 tokens
constexpr int THREADS = 320;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;
constexpr uint32_t kWaitLimit = 1u << 24;  // polls before a wait gives up (normal runs)

__device__ int g_hessian_status = 0;

// Expiry test of the bounded waits (host-set, off by default): the producer issues no load,
// so the MMA and drain warps' waits run out after `wait_limit` polls; the CTA then records
// GPTQ_ERR_TIMEOUT, frees its TMEM and returns, and H is left unchanged.
struct WaitTest {
  int skip_loads;
  uint32_t wait_limit;
};
std::atomic<int> g_test_skip{0};
std::atomic<uint32_t> g_test_limit{0};

template <uint32_t AB_FMT>
__global__ void __launch_bounds__(THREADS, 1)
    hessian_syrk_kernel(const __grid_constant__ CUtensorMap tmap, float* __restrict__ H, int n, int64_t T,
                        int tiles, int S, int64_t tok_per_seg, WaitTest wt) {
  const uint32_t WAIT_LIMIT = wt.wait_limit;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* accf = empty + STAGES;
  uint64_t* acce = accf + 2;
  uint64_t* done = acce + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = static_cast<int>(gridDim.x);
  const int units = tiles * S;  // < 2^31 (checked on the host)
  // k-steps of unit u (uniform over the CTA)
  auto unit_ksteps = [&](int u, int& tile, int64_t& t0) {
    int seg;
    hsched::unit_at(u, tiles, S, G, tile, seg);
    t0 = static_cast<int64_t>(seg) * tok_per_seg;
    const int64_t t1 = min(T, t0 + tok_per_seg);
    return t1 > t0 ? static_cast<int>((t1 - t0 + BK - 1) / BK) : 0;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accf[b], 1);
      mbar_init(&acce[b], 8);
    }
    mbar_init(done, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer
      tma_prefetch_desc(&tmap);
      int stage = 0;
      uint32_t ph = 0;
      int issued = 0;
      for (int u = blockIdx.x; u < units && ok && !wt.skip_loads; u += G) {
        int tile;
        int64_t t0;
        const int nk = unit_ksteps(u, tile, t0);
        int bi, bj;
        hsched::tile_at(tile, n, bi, bj);
        const int i0 = bi * BM, j0 = bj * BN;
        for (int ks = 0; ks < nk; ++ks) {
          if (!mbar_wait(&empty[stage], ph ^ 1u, WAIT_LIMIT)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + stage * STAGE_BYTES;
          mbar_arrive_expect_tx(&full[stage], STAGE_BYTES);
          const int y = static_cast<int>(t0 + static_cast<int64_t>(ks) * BK);
          tma_load_2d(sa, &tmap, &full[stage], i0, y);
          tma_load_2d(sa + BOX_BYTES, &tmap, &full[stage], i0 + 64, y);
#pragma unroll
          for (int q = 0; q < 4; ++q) tma_load_2d(sa + A_BYTES + q * BOX_BYTES, &tmap, &full[stage], j0 + 64 * q, y);
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            ph ^= 1u;
          }
        }
      }
      // Before leaving, make sure no copy of ours is still landing in shared memory
      // (these waits return at once on the normal path).
      for (int k = 0; k < min(issued, STAGES); ++k) {
        int s = stage - 1 - k;
        uint32_t p = ph;
        while (s < 0) {
          s += STAGES;
          p ^= 1u;
        }
        mbar_wait(&full[s], p, WAIT_LIMIT);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- UMMA issuer
      constexpr uint32_t idesc = instr_desc(AB_FMT, true, true, BM, BN);
      int stage = 0;
      uint32_t ph = 0;
      int cg = 0;  // chunks issued by this CTA so far (selects the TMEM buffer and its phase)
      for (int u = blockIdx.x; u < units && ok; u += G) {
        int tile;
        int64_t t0;
        const int nk = unit_ksteps(u, tile, t0);
        const int nchunks = (nk + FLUSH_KSTEPS - 1) / FLUSH_KSTEPS;
        int ks = 0;
        for (int c = 0; c < nchunks && ok; ++c, ++cg) {
          const int b = cg & 1;
          if (!mbar_wait(&acce[b], ((cg >> 1) & 1) ^ 1u, WAIT_LIMIT)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t dcol = tmem + static_cast<uint32_t>(b * BN);
          const int kend = min(nk, ks + FLUSH_KSTEPS);
          for (int s_in = 0; ks < kend; ++ks, ++s_in) {
            if (!mbar_wait(&full[stage], ph, WAIT_LIMIT)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sa = smem_u32(smem + stage * STAGE_BYTES);
            const uint32_t sb = sa + A_BYTES;
#pragma unroll
            for (int k = 0; k < BK / 16; ++k) {
              // 16 tokens = two 8-row swizzle atoms = 2048 bytes along K.
              const uint64_t ad = smem_desc_sw128(sa + k * 2048, BOX_BYTES, 1024);
              const uint64_t bd = smem_desc_sw128(sb + k * 2048, BOX_BYTES, 1024);
              umma_f16(dcol, ad, bd, idesc, (s_in > 0 || k > 0) ? 1u : 0u);
            }
            umma_commit(&empty[stage]);
            if (++stage == STAGES) {
              stage = 0;
              ph ^= 1u;
            }
          }
          // after a failed wait the accumulator is incomplete: never hand it to the drain
          // warps (their own bounded wait then runs out and nothing is added to H)
          if (!ok) break;
          umma_commit(&accf[b]);
        }
      }
      umma_commit(done);
      mbar_wait(done, 0, WAIT_LIMIT);
    }
  } else {
    // ---------------- accumulator drain (warps 2..9)
    const int quad = warp & 3;          // TMEM lane quarter this warp may access
    const int half = (warp - 2) >> 2;   // which 128 of the 256 columns
    float acc[128];
#pragma unroll
    for (int i = 0; i < 128; ++i) acc[i] = 0.f;
    int cg = 0;
    for (int u = blockIdx.x; u < units && ok; u += G) {
      int tile;
      int64_t t0;
      const int nk = unit_ksteps(u, tile, t0);
      const int nchunks = (nk + FLUSH_KSTEPS - 1) / FLUSH_KSTEPS;
      for (int c = 0; c < nchunks; ++c, ++cg) {
        const int b = cg & 1;
        if (!mbar_wait(&accf[b], (cg >> 1) & 1, WAIT_LIMIT)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float v[32];
          tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(quad * 32) << 16) + static_cast<uint32_t>(b * BN + half * 128 + q * 32), v);
#pragma unroll
          for (int i = 0; i < 32; ++i) acc[q * 32 + i] += v[i];
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acce[b]);
      }
      if (!ok) break;
      // Write the tile back once this CTA's next unit belongs to another tile (or there is
      // none); the MMA warp meanwhile fills the TMEM buffer just released.
      bool flush = true;
      if (u + G < units) {
        int ntile, nseg;
        hsched::unit_at(u + G, tiles, S, G, ntile, nseg);
        flush = ntile != tile;
      }
      if (!flush) continue;
      int bi, bj;
      hsched::tile_at(tile, n, bi, bj);
      const int gi = bi * BM + quad * 32 + lane;
      const int jb = bj * BN + half * 128;
      if (gi < n) {
        float* rowp = H + static_cast<size_t>(gi) * n;
#pragma unroll
        for (int c4 = 0; c4 < 32; ++c4) {
          const int gj = jb + c4 * 4;
          if (gj >= gi && gj + 3 < n) {
            atomicAdd(reinterpret_cast<float4*>(rowp + gj),
                      make_float4(2.f * acc[4 * c4], 2.f * acc[4 * c4 + 1], 2.f * acc[4 * c4 + 2], 2.f * acc[4 * c4 + 3]));
          } else {
#pragma unroll
            for (int e = 0; e < 4; ++e)
              if (gj + e < n && gj + e >= gi) atomicAdd(rowp + gj + e, 2.f * acc[4 * c4 + e]);
          }
        }
#pragma unroll
        for (int c = 0; c < 128; ++c) {
          const int gj = jb + c;
          if (gj < n && gj > gi) atomicAdd(H + static_cast<size_t>(gj) * n + gi, 2.f * acc[c]);
        }
      }
#pragma unroll
      for (int i = 0; i < 128; ++i) acc[i] = 0.f;
    }
  }
  if (!ok) atomicExch(&g_hessian_status, kStatusTimeout);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Token segments per tile.  The persistent grid runs G = min(SMs, units) CTAs; full tile
// groups take S rounds each and the last group's g*S units take ceil(g*S/G) rounds.  Pick
// the S that keeps the SMs busiest while every unit stays long enough to amortise its
// start (about ten k-steps' worth).
int choose_segments(int tiles, int64_t ksteps, int sms) {
  int best = 1;
  double best_score = -1.0;
  const int smax = static_cast<int>(std::min<int64_t>(ksteps, 1024));
  for (int S = 1; S <= smax; ++S) {
    const int64_t kper = (ksteps + S - 1) / S;
    if (S > 1 && kper < 16) break;
    const int64_t units = static_cast<int64_t>(tiles) * S;
    const int64_t G = std::min<int64_t>(sms, units);
    const int64_t full = tiles / G, g = tiles % G;
    const int64_t rounds = full * S + (g * S + G - 1) / G;
    const double eff = static_cast<double>(units) / static_cast<double>(rounds * G) *
                       static_cast<double>(G) / static_cast<double>(sms);
    const double score = eff * static_cast<double>(kper) / static_cast<double>(kper + 10);
    if (score > best_score + 1e-9) {
      best_score = score;
      best = S;
    }
  }
  return best;
}

template <uint32_t F>
int launch_impl(const void* X, int64_t T, int n, float* H, cudaStream_t st) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return GPTQ_ERR_CUDA;
  GPTQ_TRY(ensure_smem_limit(reinterpret_cast<const void*>(hessian_syrk_kernel<F>), SMEM_BYTES));
  const int tiles = hsched::tile_count(n);
  const int sms = num_sms();
  // TMA coordinates are 32-bit: walk very long token streams in chunks.
  const int64_t CH = int64_t(1) << 30;
  for (int64_t c0 = 0; c0 < T; c0 += CH) {
    const int64_t Tc = std::min(CH, T - c0);
    const char* base = static_cast<const char*>(X) + static_cast<size_t>(c0) * n * 2;
    CUtensorMap tm;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(n), static_cast<cuuint64_t>(Tc)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(n) * 2};
    cuuint32_t box[2] = {64, BK};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(&tm, F == 1 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                     const_cast<char*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return GPTQ_ERR_CUDA;
    const int64_t ksteps = (Tc + BK - 1) / BK;
    const int S0 = choose_segments(tiles, ksteps, sms);
    const int64_t tok_per_seg = ((ksteps + S0 - 1) / S0) * BK;
    const int S = static_cast<int>((Tc + tok_per_seg - 1) / tok_per_seg);  // no empty segments
    if (static_cast<int64_t>(tiles) * S >= (int64_t(1) << 31)) return GPTQ_ERR_UNSUPPORTED;
    const int G = static_cast<int>(std::min<int64_t>(sms, static_cast<int64_t>(tiles) * S));
    const uint32_t lim = g_test_limit.load();
    const WaitTest wt{g_test_skip.load(), lim ? lim : kWaitLimit};
    hessian_syrk_kernel<F><<<G, THREADS, SMEM_BYTES, st>>>(tm, H, n, Tc, tiles, S, tok_per_seg, wt);
    GPTQ_TRY(after_launch());
  }
  return GPTQ_OK;
}

}  // namespace

int launch_hessian(const void* X, int x_dtype, int64_t tokens, int64_t n, float* H, cudaStream_t s) {
  if (x_dtype == GPTQ_BF16) return launch_impl<1>(X, tokens, static_cast<int>(n), H, s);
  return launch_impl<0>(X, tokens, static_cast<int>(n), H, s);
}

void hessian_wait_test(int skip_loads, uint32_t wait_limit) {
  g_test_skip.store(skip_loads ? 1 : 0);
  g_test_limit.store(wait_limit);
}

int hessian_device_status(cudaStream_t s, int clear) {
  if (cudaStreamSynchronize(s) != cudaSuccess) return GPTQ_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_hessian_status, sizeof(int)) != cudaSuccess) return GPTQ_ERR_CUDA;
  if (clear) {
    int z = 0;
    if (cudaMemcpyToSymbol(g_hessian_status, &z, sizeof(int)) != cudaSuccess) return GPTQ_ERR_CUDA;
  }
  return v;
}

}  // namespace gptq

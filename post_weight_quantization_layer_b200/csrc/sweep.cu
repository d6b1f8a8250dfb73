// Quantize-and-compensate column sweep, lazy block updates, code packing.
//
// Source: "第5章 GPTQ 实战" §5.1.8 (the near-implementation pseudo-code): for each column
// q, quantize with the group's fixed scale, form the normalised error
// err = (w - q_int) / U[q, q], subtract err * U[q, later columns] from the columns of the
// block not yet quantized, and after each block apply all of the block's errors to the
// later columns at once as a matrix product (lazy batch update, key point 3).
// §5.1.10: each group of group_size weights of a row shares one scale and zero point.
// AutoGPTQ examples guide §1.4: sym / desc_act / static_groups.
//
// Work layout:
// * Wk [n_out, n_in] fp64 is the working copy of W in sweep order; Err [n_out, n_in] fp64
//   receives each column's normalised error, which the lazy updates read.
// * codesT [n_in, n_out] uint8 holds the codes in sweep order (column-major w.r.t. W),
//   so both the sweep's writes and the packer's reads are coalesced across rows.
// * Panels of P <= 64 columns: one kernel per panel, rows in parallel (4 threads per row,
//   16 columns per thread in registers, the panel's block of U in shared memory; per
//   column the owner's current value goes to the row's threads by one warp shuffle and
//   all of them take the decision; group min/max by warp shuffles).
// * Precision: the running weights, the errors, U and the lazy-update products are all
//   fp64; only the code decision (w / s, rounding) is taken in fp32.  GPTQ's sweep is a
//   long chain of rounding decisions, each depending on every earlier error of its row,
//   so fp32-level perturbations of the running weights grow into different codes over
//   thousands of columns.
// * Two-level lazy updates: inside an outer block (<= 512 columns) each panel kernel first
//   applies the pending errors of the block's earlier panels to its own columns (a small
//   left-looking product on the fp64 matrix units); after each outer block its errors
//   update every later column at once.  That trailing update runs on the int8 tensor cores
//   (ozaki.cu: both operands split into five 7-bit slices, exact integer slice products,
//   exact integer recombination), which leaves the fp64 pipe to the panels' compensation chain.
// * Look-ahead: the trailing update is split in two.  The next outer block's columns are
//   updated first, on a high-priority stream that then runs the next block's panels; the
//   rest runs at the same time on a low-priority stream.  A panel CTA and a trailing-update
//   CTA fit on one SM together (shared memory and registers), so the two overlap.
#include <algorithm>

#include "common.cuh"

namespace gptq {
namespace {

constexpr int PW = 64;                 // max panel width
constexpr int PTHREADS = 128;          // threads per CTA of the panel kernel
constexpr int TPR = 4;                 // threads per row
constexpr int NCOL = PW / TPR;         // columns per thread
constexpr int ROWS = PTHREADS / TPR;   // rows per CTA
// U block (fp64) + per-column reciprocal pivots (fp64) + per-column group parameters of
// every row (scale fp32, zero int32) + codes.
constexpr int KC = 32;                 // K chunk of the fused left-looking update
constexpr int EP = KC + 4, UP = PW + 4;  // padded pitches (conflict-free fragment loads)
// (the accumulated update [ROWS][UP] reuses the U staging buffers)
constexpr int PANEL_SMEM = PW * PW * 8 + PW * 8 + PW * ROWS * 8 + PW * ROWS + (2 * (ROWS * EP + KC * UP)) * 8;
static_assert(ROWS * UP <= 2 * KC * UP, "accumulator tile must fit in the staging buffers");
// Outer block width (the left-looking K inside a block stays below it), measured best on
// this part: 256 for rows of up to 6144 columns, 512 for longer rows (whose trailing GEMMs
// are large enough to amortise a wider block's panels).
int outer_block_width(int64_t n_in) { return n_in <= 6144 ? 256 : 512; }

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, bool pred) {
  const unsigned sa = static_cast<unsigned>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(sa), "l"(gmem), "r"(pred ? 16 : 0) : "memory");
}

// ---------------------------------------------------------------- quantizer (float32 decisions)
__device__ __forceinline__ void params_sym(float amax, int bits, float& s, int& z) {
  const int maxq = (1 << bits) - 1;
  const float a = (amax == 0.f) ? 1.f : amax;
  s = __fdiv_rn(__fmul_rn(2.f, a), static_cast<float>(maxq));
  z = 1 << (bits - 1);
}

__device__ __forceinline__ void params_asym(float mn, float mx, int bits, float& s, int& z) {
  const int maxq = (1 << bits) - 1;
  float lo = fminf(0.f, mn), hi = fmaxf(0.f, mx);
  if (hi == lo) {
    lo = -1.f;
    hi = 1.f;
  }
  s = __fdiv_rn(__fsub_rn(hi, lo), static_cast<float>(maxq));
  const float zf = rintf(__fdiv_rn(-lo, s));
  z = static_cast<int>(fminf(fmaxf(zf, 0.f), static_cast<float>(maxq)));
}

__device__ __forceinline__ void group_params(float mn, float mx, int bits, bool sym, float& s, int& z) {
  if (sym)
    params_sym(fmaxf(fabsf(mn), fabsf(mx)), bits, s, z);
  else
    params_asym(mn, mx, bits, s, z);
}

__device__ __forceinline__ int quant_code(float w, float s, int z, int maxq) {
  const float r = rintf(__fdiv_rn(w, s));
  const float q = fminf(fmaxf(__fadd_rn(r, static_cast<float>(z)), 0.f), static_cast<float>(maxq));
  return static_cast<int>(q);
}

__device__ __forceinline__ int64_t clamp_idx(int32_t v, int64_t n) {
  return v < 0 ? 0 : (v >= n ? n - 1 : v);
}

// ---------------------------------------------------------------- staging kernels
template <typename T>
__global__ void stage_weights_kernel(const T* __restrict__ W, int64_t n_out, int64_t n_in,
                                     const int32_t* __restrict__ perm, double* __restrict__ Wk) {
  const int64_t o = blockIdx.y;
  for (int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; j < n_in;
       j += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t c = perm ? clamp_idx(perm[j], n_in) : j;
    Wk[o * n_in + j] = static_cast<double>(to_f32(W[o * n_in + c]));
  }
}

// Parameters fixed before the sweep: group_size == -1 (whole original row) or static
// groups (consecutive original columns).  One warp per (group, row).
template <typename T>
__global__ void fixed_params_kernel(const T* __restrict__ W, int64_t n_out, int64_t n_in, int gsz, int64_t G,
                                    int bits, int sym, float* __restrict__ scales, int32_t* __restrict__ zeros) {
  const int64_t wid = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= G * n_out) return;
  const int64_t g = wid / n_out, o = wid % n_out;
  const int64_t c0 = gsz < 0 ? 0 : g * gsz;
  const int64_t c1 = gsz < 0 ? n_in : c0 + gsz;
  float mn = INFINITY, mx = -INFINITY;
  for (int64_t c = c0 + lane; c < c1; c += 32) {
    const float v = to_f32(W[o * n_in + c]);
    mn = fminf(mn, v);
    mx = fmaxf(mx, v);
  }
  for (int off = 16; off; off >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  }
  if (lane == 0) {
    float s;
    int z;
    group_params(mn, mx, bits, sym != 0, s, z);
    scales[g * n_out + o] = s;
    zeros[g * n_out + o] = z;
  }
}

// Non-static groups wider than a panel: parameters from the current (error-updated)
// weights of sweep columns [j0, j0 + gsz) when the sweep reaches j0.  One warp per row.
__global__ void current_params_kernel(const double* __restrict__ Wk, int64_t n_out, int64_t n_in, int64_t j0,
                                      int gsz, int bits, int sym, float* __restrict__ scales,
                                      int32_t* __restrict__ zeros) {
  const int64_t o = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (o >= n_out) return;
  float mn = INFINITY, mx = -INFINITY;
  for (int64_t c = j0 + lane; c < j0 + gsz; c += 32) {
    const float v = static_cast<float>(Wk[o * n_in + c]);
    mn = fminf(mn, v);
    mx = fmaxf(mx, v);
  }
  for (int off = 16; off; off >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  }
  if (lane == 0) {
    float s;
    int z;
    group_params(mn, mx, bits, sym != 0, s, z);
    scales[(j0 / gsz) * n_out + o] = s;
    zeros[(j0 / gsz) * n_out + o] = z;
  }
}

// ---------------------------------------------------------------- panel kernel
struct PanelArgs {
  double* Wk;
  double* Err;
  int64_t n_out, n_in;
  const double* U;
  int64_t j0;
  int64_t o0;  // first column of the current outer block (errors of [o0, j0) are still pending)
  int pw;
  int bits, gsz;
  int sym;
  int in_panel_params;  // 1: non-static groups that start inside this panel
  int static_groups;
  const int32_t* perm;
  float* scales;
  int32_t* zeros;
  uint8_t* codesT;
  double* loss;
};

__global__ void __launch_bounds__(PTHREADS) sweep_panel_kernel(PanelArgs a) {
  extern __shared__ __align__(16) unsigned char psm[];
  double* Us = reinterpret_cast<double*>(psm);               // [PW][PW], U[j0 + r][j0 + c]
  double* rdiag = reinterpret_cast<double*>(Us + PW * PW);   // [PW], 1 / U[j][j]
  float* ps = reinterpret_cast<float*>(rdiag + PW);          // [PW][ROWS] scale per column and row
  int* pz = reinterpret_cast<int*>(ps + PW * ROWS);          // [PW][ROWS] zero point
  uint8_t* cs = reinterpret_cast<uint8_t*>(pz + PW * ROWS);  // [PW][ROWS] codes of this CTA
  double* Es = reinterpret_cast<double*>(cs + PW * ROWS);    // [2][ROWS][EP] chunks of Err
  double* Ut = Es + 2 * ROWS * EP;                            // [2][KC][UP] chunks of U rows
  double* Cs = Ut;                                            // [ROWS][UP] accumulated update (after the loop)
  const int tid = threadIdx.x, lane = tid & 31;
  const int tsub = tid % TPR;
  const int rloc = tid / TPR;
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * ROWS;
  const int64_t row = row0 + rloc;
  const bool active = row < a.n_out;
  const int pw = a.pw;
  const int64_t j0 = a.j0, n_in = a.n_in, n_out = a.n_out;
  const int maxq = (1 << a.bits) - 1;
  const unsigned FULL = 0xffffffffu;
  const int base_lane = lane & ~(TPR - 1);

  // The panel's block of U (upper triangle): a fixed trip count, fully unrolled, so every
  // thread's loads are in flight together (each thread reads one column of 32 rows).
  static_assert((PW * PW) % PTHREADS == 0, "U block staging");
#pragma unroll
  for (int i = 0; i < PW * PW / PTHREADS; ++i) {
    const int e = tid + i * PTHREADS;
    const int r = e / PW, c = e % PW;
    Us[e] = (r < pw && c < pw && c >= r) ? a.U[(j0 + r) * n_in + j0 + c] : 0.0;
  }
  // Parameters fixed before this panel (static groups, group_size -1, or groups wider
  // than the panel): stage them per column so the serial chain below never waits on
  // global memory.
  if (!a.in_panel_params) {
    // Three phases, each with all of a thread's loads in flight together: group indices,
    // then the parameters (read-only path), then the shared-memory stores.  32-bit index
    // arithmetic (n_in < 2^16).
    int gi[NCOL];
    const int nin = static_cast<int>(n_in), jj0 = static_cast<int>(j0);
#pragma unroll
    for (int m = 0; m < NCOL; ++m) {
      const int c = tsub + TPR * m;
      const int j = jj0 + c;
      int col = j;
      if (a.static_groups && a.perm && c < pw) col = min(max(__ldg(a.perm + j), 0), nin - 1);
      gi[m] = (a.gsz > 0 && c < pw) ? col / a.gsz : 0;
    }
    float sv[NCOL];
    int zv[NCOL];
#pragma unroll
    for (int m = 0; m < NCOL; ++m) {
      const int64_t at = static_cast<int64_t>(gi[m]) * n_out + row;
      const bool ld = active && tsub + TPR * m < pw;
      sv[m] = ld ? __ldg(a.scales + at) : 1.f;
      zv[m] = ld ? __ldg(a.zeros + at) : 0;
    }
#pragma unroll
    for (int m = 0; m < NCOL; ++m) {
      const int c = tsub + TPR * m;
      if (c < pw) {
        ps[c * ROWS + rloc] = sv[m];
        pz[c * ROWS + rloc] = zv[m];
      }
    }
  }
  __syncthreads();
  if (tid < pw) rdiag[tid] = 1.0 / Us[tid * PW + tid];

  // Left-looking part of the lazy update: the errors of the earlier panels of this outer
  // block, Err[rows, o0:j0] U[o0:j0, panel], are applied here instead of by a separate
  // GEMM per panel.  fp64 on the fp64 matrix units: warp w computes columns 8w..8w+7 of
  // the 16 x 64 product as two m8n8 tiles.
  if (a.j0 > a.o0) {
    // Warp w computes rows 8w..8w+7 of the ROWS x 64 product as eight m8n8 tiles.
    const int g = lane >> 2, t = lane & 3, w = tid >> 5;
    double acc[PW / 8][2];
#pragma unroll
    for (int nb = 0; nb < PW / 8; ++nb) acc[nb][0] = acc[nb][1] = 0.0;
    const int nch = static_cast<int>((j0 - a.o0 + KC - 1) / KC);
    // 16-byte copies need even element offsets; odd panel widths (odd group sizes) take
    // the plain-load path.
    const bool vec_ok = ((j0 | a.o0 | n_in | static_cast<int64_t>(pw)) & 1) == 0;
    // Chunk ch covers error columns [o0 + ch*KC, ...); both tiles are fetched with
    // 16-byte cp.async (zero-filled outside the matrix), two chunks in flight.
    auto stage = [&](int ch, int buf) {
      const int64_t k0 = a.o0 + static_cast<int64_t>(ch) * KC;
      double* es = Es + buf * ROWS * EP;
      double* ut = Ut + buf * KC * UP;
      if (!vec_ok) {
        for (int e = tid; e < ROWS * KC; e += PTHREADS) {
          const int r = e / KC, k = e % KC;
          const int64_t gr = row0 + r, gk = k0 + k;
          es[r * EP + k] = (gr < n_out && gk < j0) ? a.Err[gr * n_in + gk] : 0.0;
        }
        for (int e = tid; e < KC * PW; e += PTHREADS) {
          const int k = e / PW, c = e % PW;
          const int64_t gk = k0 + k;
          ut[k * UP + c] = (gk < j0 && c < pw) ? a.U[gk * n_in + j0 + c] : 0.0;
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
        return;
      }
      for (int e = tid; e < ROWS * (KC / 2); e += PTHREADS) {  // rows x 16-byte chunks
        const int r = e / (KC / 2), kc = (e % (KC / 2)) * 2;
        const int64_t gr = row0 + r, gk = k0 + kc;
        const bool ok = gr < n_out && gk < j0;
        cp_async16(es + r * EP + kc, ok ? a.Err + gr * n_in + gk : a.Err, ok);
      }
      for (int e = tid; e < KC * (PW / 2); e += PTHREADS) {
        const int k = e / (PW / 2), c = (e % (PW / 2)) * 2;
        const int64_t gk = k0 + k;
        const bool ok = gk < j0 && c < pw;
        cp_async16(ut + k * UP + c, ok ? a.U + gk * n_in + j0 + c : a.U, ok);
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
    };
    stage(0, 0);
    for (int ch = 0; ch < nch; ++ch) {
      if (ch + 1 < nch) {
        stage(ch + 1, (ch + 1) & 1);
        asm volatile("cp.async.wait_group 1;" ::: "memory");
      } else {
        asm volatile("cp.async.wait_group 0;" ::: "memory");
      }
      __syncthreads();
      const double* es = Es + (ch & 1) * ROWS * EP;
      const double* ut = Ut + (ch & 1) * KC * UP;
#pragma unroll
      for (int kk = 0; kk < KC; kk += 4) {
        const double a0 = es[(w * 8 + g) * EP + kk + t];
#pragma unroll
        for (int nb = 0; nb < PW / 8; ++nb) {
          const double b0 = ut[(kk + t) * UP + nb * 8 + g];
          asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};"
                       : "+d"(acc[nb][0]), "+d"(acc[nb][1])
                       : "d"(a0), "d"(b0));
        }
      }
      __syncthreads();
    }
#pragma unroll
    for (int nb = 0; nb < PW / 8; ++nb) {
      Cs[(w * 8 + g) * UP + nb * 8 + 2 * t] = acc[nb][0];
      Cs[(w * 8 + g) * UP + nb * 8 + 2 * t + 1] = acc[nb][1];
    }
    __syncthreads();
  }
  // The panel's running weights live in registers in fp64: each column of the panel
  // receives up to PW-1 compensation updates here, and rounding the running value to
  // fp32 after each of them would push near-tie codes across a rounding boundary.  They
  // are loaded after the left-looking product, so its accumulators and these registers
  // are never live together.
  double v[NCOL];
#pragma unroll
  for (int m = 0; m < NCOL; ++m) {
    const int col = tsub + TPR * m;
    v[m] = (active && col < pw) ? a.Wk[row * n_in + j0 + col] : 0.0;
    if (a.j0 > a.o0) v[m] -= Cs[rloc * UP + col];
  }
  __syncthreads();

  float s = 1.f;
  int z = 0;
  double lsum = 0.0;

  // Column c = m * TPR + o is owned by the thread with tsub == o, in its register v[m].
  // Only the loop over m is unrolled (static register indices); the loop over o stays
  // rolled so the kernel fits the instruction cache.
#pragma unroll
  for (int m = 0; m < NCOL; ++m) {
#pragma unroll 1
    for (int o = 0; o < TPR; ++o) {
      const int c = m * TPR + o;
      if (c >= pw) break;
      const int j = static_cast<int>(j0) + c;  // < 2^16: 32-bit division below
      if (a.in_panel_params && j % a.gsz == 0) {
        float mn = INFINITY, mx = -INFINITY;
#pragma unroll
        for (int mm = m; mm < NCOL; ++mm) {
          const int col = tsub + TPR * mm;
          if (col >= c && col < c + a.gsz && col < pw) {
            const float x = static_cast<float>(v[mm]);
            mn = fminf(mn, x);
            mx = fmaxf(mx, x);
          }
        }
#pragma unroll
        for (int off = 1; off < TPR; off <<= 1) {
          mn = fminf(mn, __shfl_xor_sync(FULL, mn, off));
          mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, off));
        }
        group_params(mn, mx, a.bits, a.sym != 0, s, z);
        if (tsub == 0 && active) {
          a.scales[static_cast<int64_t>(j / a.gsz) * n_out + row] = s;
          a.zeros[static_cast<int64_t>(j / a.gsz) * n_out + row] = z;
        }
      }
      // All threads of the row take the decision on the owner's current value, so the
      // chain carries one shuffle and no divergent branch; the owner keeps the error.
      const double w = __shfl_sync(FULL, v[m], base_lane + o);
      if (!a.in_panel_params) {
        s = ps[c * ROWS + rloc];
        z = pz[c * ROWS + rloc];
      }
      const int q = quant_code(static_cast<float>(w), s, z, maxq);
      const double what = static_cast<double>(s) * static_cast<double>(q - z);
      const double err = (w - what) * rdiag[c];
      if (tsub == o) {
        v[m] = err;
        cs[c * ROWS + rloc] = static_cast<uint8_t>(q);
        lsum += err * err;
      }
      // Compensate this thread's later columns.  Only its slot m can hold a column at or
      // before c (tsub <= o); every later slot is past c.  Columns beyond the panel width
      // meet zero entries of Us and stay zero.
      const double* urow = Us + c * PW + tsub;
      if (tsub > o) v[m] = fma(-err, urow[TPR * m], v[m]);
#pragma unroll
      for (int mm = m + 1; mm < NCOL; ++mm) v[mm] = fma(-err, urow[TPR * mm], v[mm]);
    }
  }

  // errors feed the lazy updates of the later columns
#pragma unroll
  for (int m = 0; m < NCOL; ++m) {
    const int col = tsub + TPR * m;
    if (active && col < pw) a.Err[row * n_in + j0 + col] = v[m];
  }
  __syncthreads();
  // codes: one ROWS-byte row segment per column
  for (int e = tid; e < pw * ROWS; e += PTHREADS) {
    const int c = e / ROWS, r = e % ROWS;
    if (row0 + r < n_out) a.codesT[(j0 + c) * n_out + row0 + r] = cs[c * ROWS + r];
  }
  if (!active) lsum = 0.0;
  for (int off = 16; off; off >>= 1) lsum += __shfl_xor_sync(FULL, lsum, off);
  __shared__ double red[PTHREADS / 32];
  if (lane == 0) red[tid >> 5] = lsum;
  __syncthreads();
  if (tid == 0) {
    double t = 0.0;
    for (int i = 0; i < PTHREADS / 32; ++i) t += red[i];
    atomicAdd(a.loss, t);
  }
}

// ---------------------------------------------------------------- packing
// qweight[w][o]: LSB-first stream of `bits`-bit codes along the ORIGINAL column order.
// Sweep position of original column c is invperm[c].  Four outputs per thread -> one
// 128-bit store when n_out % 4 == 0.
__global__ void pack_kernel(const uint8_t* __restrict__ codesT, const int32_t* __restrict__ invperm, int64_t n_out,
                            int64_t n_in, int bits, int32_t* __restrict__ qweight) {
  const int64_t nw = n_in * bits / 32;
  const int64_t o4 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 4;
  const int64_t w = blockIdx.y;
  if (w >= nw || o4 >= n_out) return;
  const int64_t bit0 = w * 32;
  const int64_t cfirst = bit0 / bits, clast = (bit0 + 31) / bits;
  uint32_t acc[4] = {0u, 0u, 0u, 0u};
  const bool vec = (n_out % 4 == 0);
  for (int64_t c = cfirst; c <= clast && c < n_in; ++c) {
    const int64_t j = invperm ? clamp_idx(invperm[c], n_in) : c;
    const int shift = static_cast<int>(c * bits - bit0);
    uint32_t cv[4];
    if (vec) {
      const uchar4 q = *reinterpret_cast<const uchar4*>(codesT + j * n_out + o4);
      cv[0] = q.x;
      cv[1] = q.y;
      cv[2] = q.z;
      cv[3] = q.w;
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) cv[e] = (o4 + e < n_out) ? codesT[j * n_out + o4 + e] : 0u;
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t m = cv[e] & ((1u << bits) - 1u);
      acc[e] |= shift >= 0 ? (shift < 32 ? (m << shift) : 0u) : (m >> (-shift));
    }
  }
  if (vec) {
    *reinterpret_cast<int4*>(qweight + w * n_out + o4) =
        make_int4(static_cast<int>(acc[0]), static_cast<int>(acc[1]), static_cast<int>(acc[2]), static_cast<int>(acc[3]));
  } else {
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if (o4 + e < n_out) qweight[w * n_out + o4 + e] = static_cast<int32_t>(acc[e]);
  }
}

// g_idx[c] = group of original column c.
__global__ void gidx_kernel(const int32_t* __restrict__ invperm, int64_t n_in, int gsz, int static_groups,
                            int32_t* __restrict__ g_idx) {
  const int64_t c = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (c >= n_in) return;
  int64_t g = 0;
  if (gsz > 0) {
    const int64_t j = (invperm && !static_groups) ? clamp_idx(invperm[c], n_in) : c;
    g = j / gsz;
  }
  g_idx[c] = static_cast<int32_t>(g);
}

template <typename T>
int stage_and_fixed(const SweepArgs& a, cudaStream_t s) {
  const T* W = static_cast<const T*>(a.W);
  dim3 grid(static_cast<unsigned>(std::min<int64_t>((a.n_in + 255) / 256, 64)), static_cast<unsigned>(a.n_out));
  stage_weights_kernel<T><<<grid, 256, 0, s>>>(W, a.n_out, a.n_in, a.perm, a.Wk);
  GPTQ_TRY(after_launch());
  if (a.group_size < 0 || a.static_groups) {
    const int64_t G = a.group_size < 0 ? 1 : a.n_in / a.group_size;
    const int64_t warps = G * a.n_out;
    fixed_params_kernel<T><<<static_cast<unsigned>((warps * 32 + 255) / 256), 256, 0, s>>>(
        W, a.n_out, a.n_in, a.group_size, G, a.bits, a.sym ? 1 : 0, a.scales, a.zeros);
    GPTQ_TRY(after_launch());
  }
  return GPTQ_OK;
}

}  // namespace

int run_sweep(SweepArgs& a, cudaStream_t s, int* panel_width, int* outer_width) {
  GPTQ_TRY(ensure_smem_limit(reinterpret_cast<const void*>(sweep_panel_kernel), PANEL_SMEM));
  const int64_t n_out = a.n_out, n_in = a.n_in;
  const int g = a.group_size;
  const bool dynamic_groups = g > 0 && !a.static_groups;

  // Panel width: <= 128 and aligned to the groups whose parameters come from the
  // current weights, so that a group's first column always sees every earlier error.
  int P = PW;
  if (dynamic_groups) {
    if (g <= PW) {
      P = (PW / g) * g;
    } else {
      P = 1;
      for (int d = PW; d >= 1; --d)
        if (g % d == 0) {
          P = d;
          break;
        }
    }
  }
  // Outer block: a multiple of P.  When groups wider than a panel take their parameters
  // from the current weights, the outer block is the group itself, so that every earlier
  // error has reached the whole group (through the outer update) when its parameters are
  // computed at its first column.
  const int64_t Q = (dynamic_groups && g > P) ? static_cast<int64_t>(g)
                                              : static_cast<int64_t>(P) * std::max<int64_t>(1, outer_block_width(n_in) / P);
  if (panel_width) *panel_width = P;
  if (outer_width) *outer_width = static_cast<int>(std::min<int64_t>(Q, n_in));

  if (a.stats) GPTQ_CUDA(cudaEventRecord(a.ev[0], s));
  GPTQ_CUDA(cudaMemsetAsync(a.loss, 0, sizeof(double), s));
  if (a.w_dtype == GPTQ_F32)
    GPTQ_TRY(stage_and_fixed<float>(a, s));
  else if (a.w_dtype == GPTQ_F16)
    GPTQ_TRY(stage_and_fixed<__half>(a, s));
  else
    GPTQ_TRY(stage_and_fixed<__nv_bfloat16>(a, s));
  if (a.stats) GPTQ_CUDA(cudaEventRecord(a.ev[1], s));

  PanelArgs pa;
  pa.Wk = a.Wk;
  pa.Err = a.Err;
  pa.n_out = n_out;
  pa.n_in = n_in;
  pa.U = a.U;
  pa.bits = a.bits;
  pa.gsz = g;
  pa.sym = a.sym ? 1 : 0;
  pa.static_groups = a.static_groups ? 1 : 0;
  pa.perm = a.perm;
  pa.scales = a.scales;
  pa.zeros = a.zeros;
  pa.codesT = a.codesT;
  pa.loss = a.loss;
  const unsigned panel_grid = static_cast<unsigned>((n_out + ROWS - 1) / ROWS);

  // Slices of the trailing update's operands (int8 tensor cores): two sets, by outer-block
  // parity.  Block b+1 splits into the set that block b-1 used; block b-1's last reader of
  // it, its trailing GEMM on the low-priority lane, finished before block b's look-ahead
  // (which waits for it) and so before block b+1's panels and split on the panel lane.
  const int64_t KP = i8_padded_k(Q);
  const bool use_i8 = KP <= 16384;
  const int KSL = i8_slices();
  int8_t* SA[2] = {nullptr, nullptr};
  int8_t* SB[2] = {nullptr, nullptr};
  int* EA[2] = {nullptr, nullptr};
  int* EB[2] = {nullptr, nullptr};
  void* slices = nullptr;
  if (use_i8 && Q < n_in) {
    const size_t sa = (static_cast<size_t>(KSL) * n_out * KP + 255) & ~size_t(255);
    const size_t sb = (static_cast<size_t>(KSL) * n_in * KP + 255) & ~size_t(255);
    const size_t ea = (static_cast<size_t>(n_out) * 4 + 255) & ~size_t(255);
    const size_t eb = (static_cast<size_t>(n_in) * 4 + 255) & ~size_t(255);
    GPTQ_TRY(pool_alloc(&slices, 2 * (sa + sb + ea + eb), s));
    char* p = static_cast<char*>(slices);
    for (int b = 0; b < 2; ++b) {
      SA[b] = reinterpret_cast<int8_t*>(p);
      SB[b] = reinterpret_cast<int8_t*>(p + sa);
      EA[b] = reinterpret_cast<int*>(p + sa + sb);
      EB[b] = reinterpret_cast<int*>(p + sa + sb + ea);
      p += sa + sb + ea + eb;
    }
  }
  struct FreeOnExit {
    void* p;
    cudaStream_t s;
    ~FreeOnExit() { pool_free(p, s); }
  } free_slices{slices, s};  // declared before the lanes: freed after they join into s

  {
    LaneLease lanes(s);
    // panels + look-ahead (high, unless the caller runs this sweep beside more urgent work);
    // trailing update
    const LanePrio prio[2] = {a.low_priority ? kLaneLow : kLaneHigh, kLaneLow};
    GPTQ_TRY(lanes.acquire(2, prio));
    cudaStream_t sp = lanes[0].st, sg = lanes[1].st;
    cudaEvent_t pan = lanes[0].aux, rest = lanes[1].aux;
    bool rest_issued = false;
    for (int64_t O0 = 0; O0 < n_in; O0 += Q) {
      const int64_t O1 = std::min(O0 + Q, n_in);
      const int64_t O2 = std::min(O1 + Q, n_in);
      for (int64_t p0 = O0; p0 < O1; p0 += P) {
        const int64_t p1 = std::min(p0 + P, O1);
        if (dynamic_groups && g > P && p0 % g == 0) {
          current_params_kernel<<<static_cast<unsigned>((n_out * 32 + 255) / 256), 256, 0, sp>>>(
              a.Wk, n_out, n_in, p0, g, a.bits, a.sym ? 1 : 0, a.scales, a.zeros);
          GPTQ_TRY(after_launch());
        }
        pa.j0 = p0;
        pa.o0 = O0;
        pa.pw = static_cast<int>(p1 - p0);
        pa.in_panel_params = (dynamic_groups && g <= P) ? 1 : 0;
        sweep_panel_kernel<<<panel_grid, PTHREADS, PANEL_SMEM, sp>>>(pa);
        GPTQ_TRY(after_launch());
      }
      if (O1 >= n_in) break;
      // Err[:, O0:O1] is complete: every later column gets W -= Err[:, O0:O1] U[O0:O1, :].
      const int bp = static_cast<int>((O0 / Q) & 1);
      const int64_t nl = n_in - O1;  // later columns
      if (use_i8) {
        GPTQ_TRY(i8_split_rows(sp, a.Err + O0, n_in, n_out, O1 - O0, KP, SA[bp], EA[bp]));
        GPTQ_TRY(i8_split_cols(sp, a.U + O0 * n_in + O1, n_in, O1 - O0, nl, KP, SB[bp], EB[bp]));
      }
      GPTQ_CUDA(cudaEventRecord(pan, sp));
      // The next block's columns first (on the panel stream, so its panels follow at once);
      // they were last written by the previous block's trailing update.
      if (rest_issued) GPTQ_CUDA(cudaStreamWaitEvent(sp, rest, 0));
      if (use_i8)
        GPTQ_TRY(i8_gemm_sub(sp, n_out, O2 - O1, KP, SA[bp], n_out, EA[bp], SB[bp], nl, EB[bp], 0, a.Wk + O1, n_in,
                             0));
      else
        GPTQ_TRY(dgemm(sp, n_out, O2 - O1, O1 - O0, -1.0, a.Err + O0, n_in, a.U + O0 * n_in + O1, n_in, false, 1.0,
                       a.Wk + O1, n_in, false));
      // Every column after the next block, concurrently with the next block's panels.
      if (O2 < n_in) {
        GPTQ_CUDA(cudaStreamWaitEvent(sg, pan, 0));
        if (use_i8)
          GPTQ_TRY(i8_gemm_sub(sg, n_out, n_in - O2, KP, SA[bp], n_out, EA[bp], SB[bp], nl, EB[bp], O2 - O1,
                               a.Wk + O2, n_in, 0));
        else
          GPTQ_TRY(dgemm(sg, n_out, n_in - O2, O1 - O0, -1.0, a.Err + O0, n_in, a.U + O0 * n_in + O2, n_in, false,
                         1.0, a.Wk + O2, n_in, false));
        GPTQ_CUDA(cudaEventRecord(rest, sg));
        rest_issued = true;
      }
    }
  }  // joins the side streams back into s
  if (a.stats) GPTQ_CUDA(cudaEventRecord(a.ev[2], s));

  {
    const int64_t nw = n_in * a.bits / 32;
    dim3 grid(static_cast<unsigned>(((n_out + 3) / 4 + 127) / 128), static_cast<unsigned>(nw));
    pack_kernel<<<grid, 128, 0, s>>>(a.codesT, a.invperm, n_out, n_in, a.bits, a.qweight);
    GPTQ_TRY(after_launch());
    gidx_kernel<<<static_cast<unsigned>((n_in + 255) / 256), 256, 0, s>>>(a.invperm, n_in, g,
                                                                           a.static_groups ? 1 : 0, a.g_idx);
    GPTQ_TRY(after_launch());
  }
  if (a.stats) GPTQ_CUDA(cudaEventRecord(a.ev[3], s));
  return GPTQ_OK;
}

}  // namespace gptq

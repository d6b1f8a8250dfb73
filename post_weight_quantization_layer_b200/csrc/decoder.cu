// Forward pieces of a Llama-style decoder layer, for quantizing its linears in execution
// order (true_sequential).
//
// Source: AutoGPTQ examples guide §1.4 and the OLMo quick-start §三 (BaseQuantizeConfig
// field true_sequential: quantize module by module in the real execution order), §四 step 3
// (quantization runs over the model's layers on calibration data).  In execution order,
// the calibration input of each linear is produced by the layer's earlier modules with
// their weights already quantized, so the layer is run forward between quantization
// steps.  The pages do not spell the block out; the configurations name Llama-2-shaped
// layers, whose block is: h1 = h + o_proj(attn(rope(q_proj x), rope(k_proj x), v_proj x))
// with x = rmsnorm(h); h2 = h1 + down_proj(silu(gate_proj y) * up_proj y) with
// y = rmsnorm(h1).
//
// Every kernel computes in fp32 and stores 16-bit activations (rounded to nearest even),
// the precision of the calibration activations.  The linears themselves run on the
// quantized-weight kernels of w4a16.cu.
#include <algorithm>

#include "common.cuh"

namespace gptq {
namespace {

template <typename T>
__device__ __forceinline__ T st16(float v);
template <>
__device__ __forceinline__ __half st16<__half>(float v) { return __float2half_rn(v); }
template <>
__device__ __forceinline__ __nv_bfloat16 st16<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

// y = x / sqrt(mean(x^2) + eps) * gamma, one CTA per row, the sum of squares reduced in a
// fixed order.
constexpr int RN_THREADS = 256;
template <typename T>
__global__ void __launch_bounds__(RN_THREADS) rmsnorm_kernel(const T* __restrict__ x, const T* __restrict__ gamma,
                                                             int D, float eps, T* __restrict__ y) {
  const int64_t row = blockIdx.x;
  const T* xr = x + row * D;
  float s = 0.f;
  for (int i = threadIdx.x; i < D; i += RN_THREADS) {
    const float v = to_f32(xr[i]);
    s = fmaf(v, v, s);
  }
  for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  __shared__ float ws[RN_THREADS / 32];
  __shared__ float rinv;
  if ((threadIdx.x & 31) == 0) ws[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int w = 0; w < RN_THREADS / 32; ++w) t += ws[w];
    rinv = 1.f / sqrtf(t / static_cast<float>(D) + eps);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < D; i += RN_THREADS) y[row * D + i] = st16<T>(to_f32(xr[i]) * rinv * to_f32(gamma[i]));
}

// Rotary position embedding in place on [tokens, heads * d]: within each head the pairs
// (i, i + d/2), i < d/2, rotate by pos * base^(-2i/d), pos = token index within its
// sequence.  The angle and its sine and cosine are taken in double precision.
template <typename T>
__global__ void rope_kernel(T* __restrict__ x, int64_t tokens, int heads, int d, int seq_len, double base) {
  const int half = d / 2;
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= tokens * heads * half) return;
  const int c = static_cast<int>(i % half);
  const int64_t th = i / half;  // token * heads + head
  const int64_t t = th / heads;
  const double pos = static_cast<double>(t % seq_len);
  const double ang = pos * pow(base, -2.0 * c / d);
  double sn, cs;
  sincos(ang, &sn, &cs);
  T* p = x + th * d;
  const float a = to_f32(p[c]), b = to_f32(p[c + half]);
  const float fc = static_cast<float>(cs), fs = static_cast<float>(sn);
  p[c] = st16<T>(a * fc - b * fs);
  p[c + half] = st16<T>(b * fc + a * fs);
}

// Causal softmax attention per (sequence, head): O = softmax(Q K^T / sqrt(d), keys <= query)
// V.  One CTA per 64 queries of one head; key tiles of 64 staged in shared memory; online
// softmax in fp32 (running maximum and sum per query); 4 threads per query.
constexpr int AT_Q = 64, AT_K = 64, AT_THREADS = 256;
template <typename T>
__global__ void __launch_bounds__(AT_THREADS) attention_kernel(const T* __restrict__ Q, const T* __restrict__ K,
                                                               const T* __restrict__ V, int heads, int d,
                                                               int seq_len, T* __restrict__ O) {
  extern __shared__ float asm_[];
  const int dp = d + 1;
  float* Qs = asm_;               // [AT_Q][dp]
  float* Ks = Qs + AT_Q * dp;     // [AT_K][dp]
  float* Vs = Ks + AT_K * dp;     // [AT_K][dp]
  float* P = Vs + AT_K * dp;      // [AT_Q][AT_K + 1]
  const int qt = blockIdx.x, h = blockIdx.y;
  const int64_t seq0 = static_cast<int64_t>(blockIdx.z) * seq_len;
  const int64_t ld = static_cast<int64_t>(heads) * d;
  const int tid = threadIdx.x, r = tid >> 2, sub = tid & 3;
  const int q0 = qt * AT_Q;
  const int qi = q0 + r;  // query index within the sequence
  const float scale = 1.f / sqrtf(static_cast<float>(d));
  for (int e = tid; e < AT_Q * d; e += AT_THREADS) {
    const int rr = e / d, c = e % d;
    Qs[rr * dp + c] = (q0 + rr < seq_len) ? to_f32(Q[(seq0 + q0 + rr) * ld + h * d + c]) : 0.f;
  }
  float m = -INFINITY, l = 0.f;
  float acc[32];  // d / 4 <= 32
#pragma unroll
  for (int c = 0; c < 32; ++c) acc[c] = 0.f;
  const int dq = d / 4;
  const int nkt = min(qt + 1, (seq_len + AT_K - 1) / AT_K);
  for (int kt = 0; kt < nkt; ++kt) {
    const int k0 = kt * AT_K;
    __syncthreads();
    for (int e = tid; e < AT_K * d; e += AT_THREADS) {
      const int rr = e / d, c = e % d;
      const bool in = k0 + rr < seq_len;
      Ks[rr * dp + c] = in ? to_f32(K[(seq0 + k0 + rr) * ld + h * d + c]) : 0.f;
      Vs[rr * dp + c] = in ? to_f32(V[(seq0 + k0 + rr) * ld + h * d + c]) : 0.f;
    }
    __syncthreads();
    // scores of keys sub, sub + 4, ... of this tile
    float sc[AT_K / 4];
    float tmax = -INFINITY;
#pragma unroll
    for (int jj = 0; jj < AT_K / 4; ++jj) {
      const int j = jj * 4 + sub;
      float s = 0.f;
      for (int c = 0; c < d; ++c) s = fmaf(Qs[r * dp + c], Ks[j * dp + c], s);
      s *= scale;
      if (k0 + j > qi || k0 + j >= seq_len) s = -INFINITY;
      sc[jj] = s;
      tmax = fmaxf(tmax, s);
    }
    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 1));
    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 2));
    const float mnew = fmaxf(m, tmax);
    const float corr = (m == -INFINITY) ? 0.f : expf(m - mnew);
    float psum = 0.f;
#pragma unroll
    for (int jj = 0; jj < AT_K / 4; ++jj) {
      const float p = (sc[jj] == -INFINITY) ? 0.f : expf(sc[jj] - mnew);
      P[r * (AT_K + 1) + jj * 4 + sub] = p;
      psum += p;
    }
    psum += __shfl_xor_sync(0xffffffffu, psum, 1);
    psum += __shfl_xor_sync(0xffffffffu, psum, 2);
    l = l * corr + psum;
    m = mnew;
    __syncwarp();
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      if (c < dq) {
        const int col = sub * dq + c;
        float a = acc[c] * corr;
        for (int j = 0; j < AT_K; ++j) a = fmaf(P[r * (AT_K + 1) + j], Vs[j * dp + col], a);
        acc[c] = a;
      }
    }
  }
  if (qi < seq_len) {
    const float inv = 1.f / l;
#pragma unroll
    for (int c = 0; c < 32; ++c)
      if (c < dq) O[(seq0 + qi) * ld + h * d + sub * dq + c] = st16<T>(acc[c] * inv);
  }
}

// y = silu(g) * u = g / (1 + exp(-g)) * u
template <typename T>
__global__ void silu_mul_kernel(const T* __restrict__ g, const T* __restrict__ u, int64_t n, T* __restrict__ y) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float a = to_f32(g[i]);
    y[i] = st16<T>(a / (1.f + expf(-a)) * to_f32(u[i]));
  }
}

// y = a + b (the residual connection)
template <typename T>
__global__ void add_kernel(const T* __restrict__ a, const T* __restrict__ b, int64_t n, T* __restrict__ y) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    y[i] = st16<T>(to_f32(a[i]) + to_f32(b[i]));
}

unsigned ew_grid(int64_t n) { return static_cast<unsigned>(std::min<int64_t>((n + 255) / 256, 16 * 148)); }

bool is16(int dt) { return dt == GPTQ_F16 || dt == GPTQ_BF16; }

}  // namespace
}  // namespace gptq

using namespace gptq;

extern "C" int gptq_rmsnorm(const void* x, int dtype, int64_t rows, int64_t dim, const void* gamma, float eps,
                            void* y, void* stream) {
  if (!x || !gamma || !y || rows < 0 || dim <= 0 || !is16(dtype) || !(eps >= 0.f)) return GPTQ_ERR_INVALID_ARG;
  if (rows == 0) return GPTQ_OK;
  if (rows > 2147483647LL || dim > (1 << 20)) return GPTQ_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int D = static_cast<int>(dim);
  if (dtype == GPTQ_BF16)
    rmsnorm_kernel<__nv_bfloat16><<<static_cast<unsigned>(rows), RN_THREADS, 0, s>>>(
        static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(gamma), D, eps,
        static_cast<__nv_bfloat16*>(y));
  else
    rmsnorm_kernel<__half><<<static_cast<unsigned>(rows), RN_THREADS, 0, s>>>(
        static_cast<const __half*>(x), static_cast<const __half*>(gamma), D, eps, static_cast<__half*>(y));
  return after_launch();
}

extern "C" int gptq_rope(void* x, int dtype, int64_t tokens, int heads, int head_dim, int seq_len, double base,
                         void* stream) {
  if (!x || tokens < 0 || heads <= 0 || head_dim <= 0 || head_dim % 2 || seq_len <= 0 || !is16(dtype) ||
      !(base > 0.0))
    return GPTQ_ERR_INVALID_ARG;
  if (tokens == 0) return GPTQ_OK;
  const int64_t n = tokens * heads * (head_dim / 2);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const unsigned grid = static_cast<unsigned>((n + 255) / 256);
  if (dtype == GPTQ_BF16)
    rope_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(static_cast<__nv_bfloat16*>(x), tokens, heads, head_dim, seq_len,
                                                    base);
  else
    rope_kernel<__half><<<grid, 256, 0, s>>>(static_cast<__half*>(x), tokens, heads, head_dim, seq_len, base);
  return after_launch();
}

extern "C" int gptq_attention(const void* q, const void* k, const void* v, int dtype, int64_t tokens, int heads,
                              int head_dim, int seq_len, void* out, void* stream) {
  if (!q || !k || !v || !out || tokens < 0 || heads <= 0 || seq_len <= 0 || !is16(dtype)) return GPTQ_ERR_INVALID_ARG;
  if (head_dim <= 0 || head_dim % 4 || tokens % seq_len) return GPTQ_ERR_INVALID_ARG;
  if (head_dim > 128 || heads > 65535 || tokens / seq_len > 65535) return GPTQ_ERR_UNSUPPORTED;
  if (tokens == 0) return GPTQ_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int dp = head_dim + 1;
  const int smem = static_cast<int>((AT_Q * dp + 2 * AT_K * dp + AT_Q * (AT_K + 1)) * sizeof(float));
  const dim3 grid(static_cast<unsigned>((seq_len + AT_Q - 1) / AT_Q), static_cast<unsigned>(heads),
                  static_cast<unsigned>(tokens / seq_len));
  if (dtype == GPTQ_BF16) {
    GPTQ_TRY(ensure_smem_limit(reinterpret_cast<const void*>(attention_kernel<__nv_bfloat16>), smem));
    attention_kernel<__nv_bfloat16><<<grid, AT_THREADS, smem, s>>>(
        static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
        static_cast<const __nv_bfloat16*>(v), heads, head_dim, seq_len, static_cast<__nv_bfloat16*>(out));
  } else {
    GPTQ_TRY(ensure_smem_limit(reinterpret_cast<const void*>(attention_kernel<__half>), smem));
    attention_kernel<__half><<<grid, AT_THREADS, smem, s>>>(static_cast<const __half*>(q),
                                                            static_cast<const __half*>(k),
                                                            static_cast<const __half*>(v), heads, head_dim, seq_len,
                                                            static_cast<__half*>(out));
  }
  return after_launch();
}

extern "C" int gptq_silu_mul(const void* gate, const void* up, int dtype, int64_t count, void* out, void* stream) {
  if (!gate || !up || !out || count < 0 || !is16(dtype)) return GPTQ_ERR_INVALID_ARG;
  if (count == 0) return GPTQ_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype == GPTQ_BF16)
    silu_mul_kernel<__nv_bfloat16><<<ew_grid(count), 256, 0, s>>>(static_cast<const __nv_bfloat16*>(gate),
                                                                   static_cast<const __nv_bfloat16*>(up), count,
                                                                   static_cast<__nv_bfloat16*>(out));
  else
    silu_mul_kernel<__half><<<ew_grid(count), 256, 0, s>>>(static_cast<const __half*>(gate),
                                                           static_cast<const __half*>(up), count,
                                                           static_cast<__half*>(out));
  return after_launch();
}

extern "C" int gptq_add(const void* a, const void* b, int dtype, int64_t count, void* out, void* stream) {
  if (!a || !b || !out || count < 0 || !is16(dtype)) return GPTQ_ERR_INVALID_ARG;
  if (count == 0) return GPTQ_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype == GPTQ_BF16)
    add_kernel<__nv_bfloat16><<<ew_grid(count), 256, 0, s>>>(static_cast<const __nv_bfloat16*>(a),
                                                              static_cast<const __nv_bfloat16*>(b), count,
                                                              static_cast<__nv_bfloat16*>(out));
  else
    add_kernel<__half><<<ew_grid(count), 256, 0, s>>>(static_cast<const __half*>(a), static_cast<const __half*>(b),
                                                      count, static_cast<__half*>(out));
  return after_launch();
}

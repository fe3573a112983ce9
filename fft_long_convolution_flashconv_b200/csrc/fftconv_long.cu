// Causal convolution with an arbitrary real filter as long as the input
// (L up to 65536, any length), built from block convolutions of length T = 8192.
//
// H3 summary, appendix F "Raw speech and EEG": long convolutions over
// 12,000-step EEG clips; §2 "Convolutional view": y = f * u + D u with the
// causal crop of the zero-padded (linear) convolution.  A length-2L transform
// of L > 8192 does not fit one SM's shared memory in fp32, so the row is cut
// into K = ceil(L / T) blocks u_i and the filter into blocks f_j, and
//   y_m = sum_{i + j = m} low(u_i, f_j) + sum_{i + j = m - 1} high(u_i, f_j)
// where low(a, b) = causal(a, b) (the first T outputs of the linear
// convolution a * b) and high(a, b)[t] = (a * b)[T + t] (t < T - 1, and 0 at
// t = T - 1).  With ra, rb the blocks reversed in time,
//   high(a, b)[t] = causal(ra, rb)[T - 2 - t],
// so both parts come from the same fused chunk-convolution kernel
// (launch_fftconv with K chunks of T per row, fp32 I/O): for each filter
// block j one launch over all input blocks for the low parts and one over
// the reversed blocks for the high parts, accumulated in fp32, then
// y = acc + D u rounded once to the I/O type.
#include "kernels.cuh"

namespace fc {

namespace {
constexpr int kBT = 8192;  // block length
constexpr int kThr = 256;

template <typename T> __device__ __forceinline__ float ld_io(const T* p) { return (float)*p; }
template <> __device__ __forceinline__ float ld_io<__half>(const __half* p) { return __half2float(*p); }
template <> __device__ __forceinline__ float ld_io<__nv_bfloat16>(const __nv_bfloat16* p) { return __bfloat162float(*p); }
template <typename T> __device__ __forceinline__ T st_io(float v) { return (T)v; }
template <> __device__ __forceinline__ __half st_io<__half>(float v) { return __float2half_rn(v); }
template <> __device__ __forceinline__ __nv_bfloat16 st_io<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

// U[r][t] = u[r][t] (0 for t >= L), Ur = the same with every block reversed; rows of K T floats.
template <typename T>
__global__ void __launch_bounds__(kThr) lc_stage_u(const T* __restrict__ u, float* __restrict__ U,
                                                   float* __restrict__ Ur, long long rows, int L, int K) {
  const long long KT = (long long)K * kBT;
  for (long long e = blockIdx.x * (long long)kThr + threadIdx.x; e < rows * KT; e += (long long)gridDim.x * kThr) {
    const long long r = e / KT;
    const int t = (int)(e - r * KT);
    const float v = t < L ? ld_io(u + r * L + t) : 0.f;
    const int i = t / kBT, p = t - i * kBT;
    U[e] = v;
    Ur[r * KT + (long long)i * kBT + (kBT - 1 - p)] = v;
  }
}

// F[j][h][p] = f[h][j T + p] (0 past L), Fr[j][h] = F[j][h] reversed.
__global__ void __launch_bounds__(kThr) lc_stage_f(const float* __restrict__ f, float* __restrict__ F,
                                                   float* __restrict__ Fr, int H, int L, int K) {
  const long long n = (long long)K * H * kBT;
  for (long long e = blockIdx.x * (long long)kThr + threadIdx.x; e < n; e += (long long)gridDim.x * kThr) {
    const long long jh = e / kBT;
    const int p = (int)(e - jh * kBT);
    const int j = (int)(jh / H), h = (int)(jh - (long long)j * H);
    const int t = j * kBT + p;
    const float v = t < L ? f[(long long)h * L + t] : 0.f;
    F[e] = v;
    Fr[jh * kBT + (kBT - 1 - p)] = v;
  }
}

// acc block i + j (+1 for the high parts) += the block-i result of filter block j.
__global__ void __launch_bounds__(kThr) lc_accumulate(float* __restrict__ acc, const float* __restrict__ tmp,
                                                      long long rows, int K, int j, int high) {
  const long long KT = (long long)K * kBT;
  for (long long e = blockIdx.x * (long long)kThr + threadIdx.x; e < rows * KT; e += (long long)gridDim.x * kThr) {
    const long long r = e / KT;
    const int t = (int)(e - r * KT);
    const int m = t / kBT, p = t - m * kBT;  // destination block and position
    const int i = m - j - high;              // source block
    if (i < 0) continue;
    if (!high) {
      acc[e] += tmp[r * KT + (long long)i * kBT + p];
    } else if (p <= kBT - 2) {
      acc[e] += tmp[r * KT + (long long)i * kBT + (kBT - 2 - p)];
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(kThr) lc_finalize(const float* __restrict__ acc, const T* __restrict__ u,
                                                    const float* __restrict__ D, T* __restrict__ y, long long rows,
                                                    int H, int L, int K) {
  const long long KT = (long long)K * kBT;
  for (long long e = blockIdx.x * (long long)kThr + threadIdx.x; e < rows * L; e += (long long)gridDim.x * kThr) {
    const long long r = e / L;
    const int t = (int)(e - r * L);
    const int h = (int)(r % H);
    y[e] = st_io<T>(acc[r * KT + t] + D[h] * ld_io(u + e));
  }
}

size_t round256(size_t b) { return (b + 255) & ~(size_t)255; }

int grid_for(long long n) {
  const long long g = (n + kThr - 1) / kThr;
  const long long cap = (long long)num_sms() * 16;
  return (int)(g < cap ? g : cap);
}

template <typename T>
cudaError_t long_conv_t(const void* u, const float* f, const float* D, void* y, int B, int H, int L, char* ws,
                        int dtype, cudaStream_t st) {
  const int K = (L + kBT - 1) / kBT;
  const long long rows = (long long)B * H, KT = (long long)K * kBT;
  const size_t row_bytes = round256((size_t)rows * KT * sizeof(float));
  const size_t fil_bytes = round256((size_t)K * H * kBT * sizeof(float));
  float* U = (float*)ws;
  float* Ur = (float*)(ws + row_bytes);
  float* tmp = (float*)(ws + 2 * row_bytes);
  float* acc = (float*)(ws + 3 * row_bytes);
  float* F = (float*)(ws + 4 * row_bytes);
  float* Fr = (float*)(ws + 4 * row_bytes + fil_bytes);
  float* zeroD = (float*)(ws + 4 * row_bytes + 2 * fil_bytes);
  cudaError_t e;
  if ((e = cudaMemsetAsync(acc, 0, (size_t)rows * KT * sizeof(float), st)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(zeroD, 0, (size_t)H * sizeof(float), st)) != cudaSuccess) return e;
  lc_stage_u<T><<<grid_for(rows * KT), kThr, 0, st>>>((const T*)u, U, Ur, rows, L, K);
  lc_stage_f<<<grid_for((long long)K * H * kBT), kThr, 0, st>>>(f, F, Fr, H, L, K);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const SsmArgs none{nullptr, nullptr, nullptr, nullptr, 0};
  for (int j = 0; j < K; ++j) {
    for (int high = 0; high < 2; ++high) {
      if (high && j + 1 >= K) continue;  // the high parts of filter block j land in blocks >= j + 1
      e = launch_fftconv(high ? Ur : U, (high ? Fr : F) + (size_t)j * H * kBT, kBT, none, zeroD, tmp, B, H, KT, kBT,
                         K, /*dtype=*/0, st);
      if (e != cudaSuccess) return e;
      lc_accumulate<<<grid_for(rows * KT), kThr, 0, st>>>(acc, tmp, rows, K, j, high);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
  }
  lc_finalize<T><<<grid_for(rows * L), kThr, 0, st>>>(acc, (const T*)u, D, (T*)y, rows, H, L, K);
  (void)dtype;
  return cudaGetLastError();
}
}  // namespace

size_t fftconv_long_workspace_bytes(int B, int H, int L) {
  const int K = (L + kBT - 1) / kBT;
  const long long rows = (long long)B * H, KT = (long long)K * kBT;
  return 4 * round256((size_t)rows * KT * sizeof(float)) + 2 * round256((size_t)K * H * kBT * sizeof(float)) +
         round256((size_t)H * sizeof(float));
}

cudaError_t launch_fftconv_long(const void* u, const float* f, const float* D, void* y, int B, int H, int L,
                                void* workspace, int dtype, cudaStream_t st) {
  char* ws = (char*)workspace;
  switch (dtype) {
    case 0: return long_conv_t<float>(u, f, D, y, B, H, L, ws, dtype, st);
    case 1: return long_conv_t<__half>(u, f, D, y, B, H, L, ws, dtype, st);
    default: return long_conv_t<__nv_bfloat16>(u, f, D, y, B, H, L, ws, dtype, st);
  }
}

}  // namespace fc

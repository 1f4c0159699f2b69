// Exhaustive checks of two device helpers of the row-wise append kernel, run by
// tests/test_gpu_rounding_helpers.py:
//  * div7_rn(a) (Markstein's division by 7) against the IEEE division __fdiv_rn(a, 7)
//    for every finite a >= 0 (bit patterns 0 .. 0x7f7fffff);
//  * rcp_approx(s) against the exact reciprocal (binary64) for every positive
//    binary16 normal s, as a relative error in units of 2^-23.
// Prints one JSON line.
#include <cstdio>
#include <cstring>

#include "../../compressed_domain_attention_b200/csrc/tq_device.cuh"

__device__ unsigned long long g_bad;
__device__ unsigned int g_first_bad;
__device__ unsigned int g_max_err_bits;  // binary32 bits of the largest relative error x 2^23

__global__ void check_div7(unsigned int base) {
  const unsigned int i = base + blockIdx.x * blockDim.x + threadIdx.x;
  if (i > 0x7f7fffffu) return;
  const float a = __uint_as_float(i);
  if (__float_as_uint(tqk::div7_rn(a)) != __float_as_uint(__fdiv_rn(a, 7.0f))) {
    if (atomicAdd(&g_bad, 1ull) == 0ull) g_first_bad = i;
  }
}

__global__ void check_rcp() {
  const unsigned int h = 0x0400u + blockIdx.x * blockDim.x + threadIdx.x;  // binary16 normals
  if (h > 0x7BFFu) return;
  const float s = __half2float(__ushort_as_half((unsigned short)h));
  const double exact = 1.0 / (double)s;
  const double rel = fabs((double)tqk::rcp_approx(s) - exact) / exact;
  atomicMax(&g_max_err_bits, __float_as_uint((float)(rel * 8388608.0)));
}

int main() {
  for (unsigned long long base = 0; base <= 0x7f7fffffull; base += (1ull << 28))
    check_div7<<<(unsigned)((1ull << 28) / 256), 256>>>((unsigned int)base);
  check_rcp<<<(0x7BFF - 0x0400 + 256) / 256, 256>>>();
  const cudaError_t e = cudaDeviceSynchronize();
  unsigned long long bad = 0;
  unsigned int first = 0, mx = 0;
  cudaMemcpyFromSymbol(&bad, g_bad, sizeof(bad));
  cudaMemcpyFromSymbol(&first, g_first_bad, sizeof(first));
  cudaMemcpyFromSymbol(&mx, g_max_err_bits, sizeof(mx));
  float mxf;
  std::memcpy(&mxf, &mx, sizeof(mxf));
  std::printf("{\"cuda\": \"%s\", \"div7_checked\": %u, \"div7_mismatches\": %llu, \"first_mismatch\": %u, "
              "\"rcp_max_rel_err_ulp23\": %.6f}\n",
              cudaGetErrorString(e), 0x7f800000u, bad, first, mxf);
  return e == cudaSuccess ? 0 : 1;
}

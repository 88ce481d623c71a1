// Exhaustive GPU check of the FP8 scale arithmetic of the kernels
// (csrc/quant.cuh) against CUDA's IEEE operations, for every positive finite
// bf16 and binary16 amax:
//   scale_div448(amax) == __fdiv_rn(amax, 448)          (bit for bit)
//   recip_down(s) is RN(1/s) or one ulp below it, and s * recip_down(s) <= 1
//   (exact residual not negative) for s >= 2^-120
// (the E4M3 quotient is proven on the CPU for every r within one ulp of
// RN(1/s), tests/quotient_proof.c).  Prints the counts; exits 0 iff clean.
#include <cstdio>

#include "quant.cuh"

using namespace fn;

__global__ void check(int fp16, unsigned long long* bad_scale, unsigned long long* bad_recip,
                      unsigned long long* checked, int* max_ulp) {
  const uint32_t ab = blockIdx.x * blockDim.x + threadIdx.x + 1;
  const uint32_t end = fp16 ? 0x7C00u : 0x7F80u;
  if (ab >= end) return;
  const float amax = fp16 ? f16_lo(ab) : bf_lo(ab);
  const float s_ref = __fdiv_rn(amax, 448.f);
  const float s = scale_div448(amax);
  if (__float_as_uint(s) != __float_as_uint(s_ref)) atomicAdd(bad_scale, 1ull);
  if (s_ref >= 0x1p-120f) {
    const float r_ref = __frcp_rn(s_ref), r = recip_down(s_ref);
    const int d = (int)__float_as_uint(r_ref) - (int)__float_as_uint(r);
    atomicMax(max_ulp, abs(d));
    if (d < 0 || d > 1 || fmaf(-s_ref, r, 1.0f) < 0.f) atomicAdd(bad_recip, 1ull);
    atomicAdd(checked, 1ull);
  }
}

int main() {
  unsigned long long* c;
  int* m;
  if (cudaMalloc(&c, 3 * sizeof(unsigned long long)) != cudaSuccess ||
      cudaMalloc(&m, sizeof(int)) != cudaSuccess)
    return 2;
  int rc = 0;
  for (int fp16 = 0; fp16 < 2; ++fp16) {
    cudaMemset(c, 0, 3 * sizeof(unsigned long long));
    cudaMemset(m, 0, sizeof(int));
    check<<<(0x7F80 + 255) / 256, 256>>>(fp16, c, c + 1, c + 2, m);
    unsigned long long h[3];
    int hm = 0;
    if (cudaMemcpy(h, c, sizeof h, cudaMemcpyDeviceToHost) != cudaSuccess ||
        cudaMemcpy(&hm, m, sizeof hm, cudaMemcpyDeviceToHost) != cudaSuccess)
      return 2;
    printf("%s: scale mismatches %llu, reciprocals checked %llu, bad reciprocals %llu, max ulp %d\n",
           fp16 ? "fp16" : "bf16", h[0], h[2], h[1], hm);
    if (h[0] || h[1] || h[2] == 0) rc = 1;
  }
  cudaFree(c);
  cudaFree(m);
  return rc;
}

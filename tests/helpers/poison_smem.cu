// Test helper (not part of the library): fills the dynamic shared memory of one
// CTA per SM with a byte pattern and exits.  Shared memory is not cleared
// between kernels, so a kernel launched right after finds the pattern in any
// shared memory it reads before writing; 0xFF bytes are NaN as fp16 and fp32.
#include <cuda_runtime.h>
#include <stdint.h>

__global__ void poison_smem_kernel(uint32_t words, uint32_t value) {
  extern __shared__ uint32_t s[];
  for (uint32_t i = threadIdx.x; i < words; i += blockDim.x) s[i] = value;
  __syncthreads();
  // keep the stores: a value the compiler cannot prove unread
  if (threadIdx.x == 0 && s[words - 1] == 0x12345678u && value != 0x12345678u) s[0] = 0;
}

extern "C" int poison_smem(int blocks, int bytes, uint32_t value, cudaStream_t stream) {
  if (blocks <= 0 || bytes < 4) return 1;
  if (cudaFuncSetAttribute(poison_smem_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           bytes) != cudaSuccess)
    return 2;
  poison_smem_kernel<<<blocks, 1024, bytes, stream>>>(static_cast<uint32_t>(bytes / 4), value);
  return cudaGetLastError() == cudaSuccess ? 0 : 3;
}

// Seeded synthetic input generator, device side.
//
// Fills device buffers with the same values as synth_cpu.c, from the same
// published definition (Philox4x32-10, Salmon et al., SC'11; Irwin-Hall sum of
// eight 16-bit uniforms; one fp32 multiply, one fp32 add, bf16 round to nearest
// even). Written separately from the host file; the two are checked for bitwise
// equality by the test suite. Used only to materialise large inputs (weights,
// cached K/V) directly in HBM; it computes nothing of the serving iteration.
#include <cstdint>
#include <cuda_runtime.h>

namespace {

__device__ __forceinline__ void philox10(uint32_t& c0, uint32_t& c1, uint32_t& c2, uint32_t& c3,
                                         uint32_t k0, uint32_t k1) {
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        const uint32_t lo0 = 0xD2511F53u * c0;
        const uint32_t hi0 = __umulhi(0xD2511F53u, c0);
        const uint32_t lo1 = 0xCD9E8D57u * c2;
        const uint32_t hi1 = __umulhi(0xCD9E8D57u, c2);
        const uint32_t n0 = hi1 ^ c1 ^ k0;
        const uint32_t n2 = hi0 ^ c3 ^ k1;
        c0 = n0; c1 = lo1; c2 = n2; c3 = lo0;
        k0 += 0x9E3779B9u;
        k1 += 0xBB67AE85u;
    }
}

__device__ __forceinline__ uint16_t normal_bf16_at(uint32_t seed, uint32_t tid, uint64_t i,
                                                   float scale, float mean) {
    uint32_t c0 = (uint32_t)i, c1 = (uint32_t)(i >> 32), c2 = 0u, c3 = 0u;
    philox10(c0, c1, c2, c3, seed, tid);
    int32_t s = (int32_t)(c0 & 0xFFFFu) + (int32_t)(c0 >> 16) + (int32_t)(c1 & 0xFFFFu) +
                (int32_t)(c1 >> 16) + (int32_t)(c2 & 0xFFFFu) + (int32_t)(c2 >> 16) +
                (int32_t)(c3 & 0xFFFFu) + (int32_t)(c3 >> 16);
    float t = __fmul_rn((float)(s - 262140), scale);
    float v = __fadd_rn(t, mean);
    uint32_t u = __float_as_uint(v);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

__global__ void fill_normal_bf16_kernel(uint32_t seed, uint32_t tid, uint64_t offset, uint64_t n,
                                        float scale, float mean, uint16_t* __restrict__ out) {
    const uint64_t stride = (uint64_t)gridDim.x * blockDim.x * 4;
    for (uint64_t j = ((uint64_t)blockIdx.x * blockDim.x + threadIdx.x) * 4; j < n; j += stride) {
        if (j + 4 <= n && ((reinterpret_cast<uintptr_t>(out + j) & 7u) == 0)) {
            uint16_t a = normal_bf16_at(seed, tid, offset + j + 0, scale, mean);
            uint16_t b = normal_bf16_at(seed, tid, offset + j + 1, scale, mean);
            uint16_t c = normal_bf16_at(seed, tid, offset + j + 2, scale, mean);
            uint16_t d = normal_bf16_at(seed, tid, offset + j + 3, scale, mean);
            uint2 pk;
            pk.x = (uint32_t)a | ((uint32_t)b << 16);
            pk.y = (uint32_t)c | ((uint32_t)d << 16);
            *reinterpret_cast<uint2*>(out + j) = pk;
        } else {
            for (uint64_t e = j; e < n && e < j + 4; ++e)
                out[e] = normal_bf16_at(seed, tid, offset + e, scale, mean);
        }
    }
}

}  // namespace

extern "C" int nfs_gpu_fill_normal_bf16(uint32_t seed, uint32_t tid, uint64_t offset, uint64_t n,
                                        float scale, float mean, void* out, void* stream) {
    if (n == 0) return 0;
    if (out == nullptr) return (int)cudaErrorInvalidValue;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    uint64_t want = (n + 4 * 256 - 1) / (4 * 256);
    uint64_t cap = (uint64_t)sms * 8;
    unsigned grid = (unsigned)(want < cap ? want : cap);
    fill_normal_bf16_kernel<<<grid, 256, 0, (cudaStream_t)stream>>>(seed, tid, offset, n, scale, mean,
                                                                   (uint16_t*)out);
    return (int)cudaGetLastError();
}

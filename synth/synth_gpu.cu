// GPU copy of the seeded normal generator in synth.c (Philox4x32-10 counter
// stream, Box-Muller in fp64), for filling benchmark-sized weight tensors in
// device memory. Test and benchmark infrastructure; holds none of the layer's
// arithmetic. Integer stages match the host bit for bit; fp64 log/sin/cos may
// differ from the host libm in the last place, which after rounding to fp32
// changes a value very rarely. Anything the oracle consumes comes from the
// host generator.
#include <cuda_runtime.h>
#include <stdint.h>

__device__ __forceinline__ void philox10(uint32_t x[4], uint32_t k0, uint32_t k1) {
    for (int r = 0; r < 10; ++r) {
        if (r) {
            k0 += 0x9E3779B9u;
            k1 += 0xBB67AE85u;
        }
        const uint32_t hi0 = __umulhi(0xD2511F53u, x[0]), lo0 = 0xD2511F53u * x[0];
        const uint32_t hi1 = __umulhi(0xCD9E8D57u, x[2]), lo1 = 0xCD9E8D57u * x[2];
        const uint32_t y0 = hi1 ^ x[1] ^ k0, y2 = hi0 ^ x[3] ^ k1;
        x[0] = y0;
        x[1] = lo1;
        x[2] = y2;
        x[3] = lo0;
    }
}

__device__ __forceinline__ double u53(uint32_t hi, uint32_t lo) {
    const uint64_t v = (((uint64_t)hi << 32) | lo) >> 11;
    return ((double)v + 0.5) * 0x1.0p-53;
}

__global__ void normal_f32_kernel(uint64_t seed, uint32_t tensor, uint32_t sub, uint64_t first, int64_t n,
                                  double mean, double std, float *out) {
    const uint64_t b0 = first >> 1;
    const int64_t nb = (int64_t)(((first + (uint64_t)n + 1) >> 1) - b0);
    for (int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; q < nb; q += (int64_t)gridDim.x * blockDim.x) {
        const uint64_t b = b0 + (uint64_t)q;
        uint32_t x[4] = {(uint32_t)b, (uint32_t)(b >> 32), sub, 0u};
        philox10(x, (uint32_t)seed, tensor ^ (uint32_t)(seed >> 32));
        const double rad = sqrt(-2.0 * log(u53(x[0], x[1])));
        const double ang = 6.283185307179586476925286766559 * u53(x[2], x[3]);
        const double z[2] = {rad * cos(ang), rad * sin(ang)};
        for (int h = 0; h < 2; ++h) {
            const int64_t i = (int64_t)(2 * b + h) - (int64_t)first;
            if (i >= 0 && i < n) out[i] = (float)(mean + std * z[h]);
        }
    }
}

extern "C" __attribute__((visibility("default"))) int synth_gpu_normal_f32(
    uint64_t seed, uint32_t tensor, uint32_t sub, uint64_t first, int64_t n, double mean, double std,
    float *out, void *stream) {
    if (n <= 0) return 0;
    normal_f32_kernel<<<1184, 256, 0, static_cast<cudaStream_t>(stream)>>>(seed, tensor, sub, first, n, mean,
                                                                           std, out);
    return (int)cudaGetLastError();
}

// Device twin of synth.c: the same counter-based SplitMix64 + Box-Muller
// generator, written a second time for the GPU so that multi-gigabyte
// synthetic weights can be made in device memory. It holds no layer
// arithmetic. The host definitions in synth.c are the specification; a GPU
// test compares both on sampled indices.
#include <cstdint>
#include <cuda_runtime.h>

namespace {

constexpr uint64_t kG = 0x9E3779B97F4A7C15ULL;

__host__ __device__ inline uint64_t mix(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

__host__ __device__ inline uint64_t stream_key(uint64_t seed, uint64_t id) {
    return mix(mix(seed + kG) ^ (id * kG + 1ULL));
}

__device__ inline uint64_t raw(uint64_t key, uint64_t n) { return mix(key + (n + 1ULL) * kG); }

// fp64 -> bf16 bits, nearest-even, by the same frexp / scale / rint steps as the host.
__device__ inline uint16_t round_bf16(double v) {
    if (v == 0.0) return signbit(v) ? 0x8000u : 0u;
    int e;
    double m = frexp(fabs(v), &e);
    (void)m;
    int q = e - 8;
    if (q < -133) q = -133;
    double r = rint(ldexp(fabs(v), -q));
    float f = (float)ldexp(r, q);
    uint16_t h = (uint16_t)(__float_as_uint(f) >> 16);
    if (v < 0) h |= 0x8000u;
    return h;
}

__device__ inline double normal(uint64_t key, uint64_t i) {
    uint64_t j = i >> 1;
    uint64_t a = raw(key, 2 * j), b = raw(key, 2 * j + 1);
    double u1 = (double)((a >> 11) + 1ULL) * 0x1.0p-53;
    double u2 = (double)(b >> 11) * 0x1.0p-53;
    double r = sqrt(-2.0 * log(u1));
    double t = 6.283185307179586476925286766559 * u2;
    return (i & 1ULL) ? r * sin(t) : r * cos(t);
}

__global__ void fill_bf16_kernel(uint16_t* out, int64_t n, uint64_t key, double mean, double std) {
    int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
        out[i] = round_bf16(mean + std * normal(key, (uint64_t)i));
}

__global__ void fill_bf16_as_f32_kernel(float* out, int64_t n, uint64_t key, double mean, double std) {
    int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
        out[i] = __uint_as_float((uint32_t)round_bf16(mean + std * normal(key, (uint64_t)i)) << 16);
}

__global__ void fill_i8_kernel(int8_t* out, int64_t n, uint64_t key, double std) {
    int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
        double v = rint(std * normal(key, (uint64_t)i));
        v = v > 127.0 ? 127.0 : (v < -127.0 ? -127.0 : v);
        out[i] = (int8_t)v;
    }
}

}  // namespace

extern "C" {

// out (device, int8 [n]) = clamp(nearbyint(std * z_i), -127, 127) for stream (seed, id).
int syn_dev_fill_i8(void* out, int64_t n, uint64_t seed, uint64_t id, double std, cudaStream_t stream) {
    if (n <= 0) return 0;
    int blocks = (int)((n + 255) / 256);
    if (blocks > 148 * 32) blocks = 148 * 32;
    fill_i8_kernel<<<blocks, 256, 0, stream>>>((int8_t*)out, n, stream_key(seed, id), std);
    return (int)cudaGetLastError();
}

// out (device, bf16 bits [n]) = bf16(mean + std * z_i) for stream (seed, id). Returns cudaError_t.
int syn_dev_fill_bf16(void* out, int64_t n, uint64_t seed, uint64_t id, double mean, double std,
                      cudaStream_t stream) {
    if (n <= 0) return 0;
    int blocks = (int)((n + 255) / 256);
    if (blocks > 148 * 32) blocks = 148 * 32;
    fill_bf16_kernel<<<blocks, 256, 0, stream>>>((uint16_t*)out, n, stream_key(seed, id), mean, std);
    return (int)cudaGetLastError();
}

// Same values widened to fp32 (1-D parameters).
int syn_dev_fill_bf16_as_f32(float* out, int64_t n, uint64_t seed, uint64_t id, double mean, double std,
                             cudaStream_t stream) {
    if (n <= 0) return 0;
    int blocks = (int)((n + 255) / 256);
    if (blocks > 148 * 32) blocks = 148 * 32;
    fill_bf16_as_f32_kernel<<<blocks, 256, 0, stream>>>(out, n, stream_key(seed, id), mean, std);
    return (int)cudaGetLastError();
}

}  // extern "C"

// GPU side of the seeded input generator (see synth/fill.py for the definition).  Element e
// of a tensor draws r_e, the e-th output of SplitMix64 seeded with `key`; the four 16-bit
// lanes of r_e sum to an Irwin-Hall(4) integer n_e, centred by 131070; the value is
// bf16_rne(float32(n_e) * scale).  The CPU generator produces the same bits.
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace {

__device__ __forceinline__ uint16_t value_at(uint64_t key, float scale, uint64_t e) {
    uint64_t z = key + (e + 1ull) * 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    z ^= z >> 31;
    const int32_t s = static_cast<int32_t>((z & 0xFFFF) + ((z >> 16) & 0xFFFF) + ((z >> 32) & 0xFFFF) + (z >> 48));
    const float f = __fmul_rn(static_cast<float>(s - 131070), scale);
    return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

__global__ void fill_kernel(uint16_t *dst, uint64_t n, uint64_t offset, uint64_t key, float scale) {
    const uint64_t stride = static_cast<uint64_t>(gridDim.x) * blockDim.x;
    const uint64_t n8 = n / 8;
    for (uint64_t i = static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8; i += stride) {
        uint32_t w[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint64_t e = offset + i * 8 + 2 * j;
            w[j] = static_cast<uint32_t>(value_at(key, scale, e)) |
                   (static_cast<uint32_t>(value_at(key, scale, e + 1)) << 16);
        }
        reinterpret_cast<uint4 *>(dst)[i] = make_uint4(w[0], w[1], w[2], w[3]);
    }
    for (uint64_t i = n8 * 8 + static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride)
        dst[i] = value_at(key, scale, offset + i);
}

// e4m3 code of n / 2^13 (|n| < 2^17), round to nearest even -- the integer steps of
// synth.fill.encode_e4m3_int.
__device__ __forceinline__ uint8_t encode_e4m3_int(int32_t n) {
    const uint32_t a = static_cast<uint32_t>(n < 0 ? -n : n);
    if (a == 0) return 0;
    const uint32_t sign = n < 0 ? 0x80u : 0u;
    const int msb = 31 - __clz(a);
    const int e = msb - 13;
    uint32_t code;
    if (e >= -6) {
        const int sh = msb - 3 > 0 ? msb - 3 : 0;
        uint32_t q = a >> sh;
        if (sh > 0) {
            const uint32_t rem = a - (q << sh), half = 1u << (sh - 1);
            if (rem > half || (rem == half && (q & 1u))) ++q;
        }
        int en = e;
        if (q == 16) {
            q = 8;
            ++en;
        }
        code = (static_cast<uint32_t>(en + 7) << 3) | (q - 8);
    } else {
        uint32_t q = a >> 4;
        const uint32_t r = a & 15u;
        if (r > 8 || (r == 8 && (q & 1u))) ++q;
        code = q;
    }
    return static_cast<uint8_t>(code | sign);
}

__device__ __forceinline__ uint8_t fp8_at(uint64_t key, uint64_t e) {
    uint64_t z = key + (e + 1ull) * 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    z ^= z >> 31;
    const int32_t s = static_cast<int32_t>((z & 0xFFFF) + ((z >> 16) & 0xFFFF) + ((z >> 32) & 0xFFFF) + (z >> 48));
    return encode_e4m3_int(s - 131070);
}

__global__ void fill_fp8_kernel(uint8_t *dst, uint64_t n, uint64_t offset, uint64_t key) {
    const uint64_t stride = static_cast<uint64_t>(gridDim.x) * blockDim.x;
    const uint64_t n16 = n / 16;
    for (uint64_t i = static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n16; i += stride) {
        uint32_t w[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint64_t e = offset + i * 16 + 4 * j;
            w[j] = static_cast<uint32_t>(fp8_at(key, e)) | (static_cast<uint32_t>(fp8_at(key, e + 1)) << 8) |
                   (static_cast<uint32_t>(fp8_at(key, e + 2)) << 16) | (static_cast<uint32_t>(fp8_at(key, e + 3)) << 24);
        }
        reinterpret_cast<uint4 *>(dst)[i] = make_uint4(w[0], w[1], w[2], w[3]);
    }
    for (uint64_t i = n16 * 16 + static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride)
        dst[i] = fp8_at(key, offset + i);
}

}  // namespace

extern "C" {

// dst: device or mapped memory holding n e4m3 codes (16-byte aligned).
int synth_fill_fp8(void *dst, uint64_t n, uint64_t offset, uint64_t key, void *stream) {
    if (n == 0) return 0;
    if (dst == nullptr || (reinterpret_cast<uintptr_t>(dst) & 15u)) return static_cast<int>(cudaErrorInvalidValue);
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    uint64_t blocks = (n / 16 + 255) / 256;
    const uint64_t cap = static_cast<uint64_t>(sms) * 16;
    if (blocks > cap) blocks = cap;
    if (blocks == 0) blocks = 1;
    fill_fp8_kernel<<<static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<uint8_t *>(dst), n, offset, key);
    return static_cast<int>(cudaGetLastError());
}


// dst: device or mapped memory holding n bf16 values (16-byte aligned).  Element i of dst
// receives generator element offset + i.  Returns a cudaError_t code (0 = success).
int synth_fill_bf16(void *dst, uint64_t n, uint64_t offset, uint64_t key, float scale, void *stream) {
    if (n == 0) return 0;
    if (dst == nullptr || (reinterpret_cast<uintptr_t>(dst) & 15u)) return static_cast<int>(cudaErrorInvalidValue);
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    uint64_t blocks = (n / 8 + 255) / 256;
    const uint64_t cap = static_cast<uint64_t>(sms) * 16;
    if (blocks > cap) blocks = cap;
    if (blocks == 0) blocks = 1;
    fill_kernel<<<static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<uint16_t *>(dst), n, offset, key, scale);
    return static_cast<int>(cudaGetLastError());
}

// Pinned host memory mapped into the device address space (for host-resident tables).
// Returns a cudaError_t code; *out receives a pointer usable from host and device.
int synth_host_alloc_mapped(uint64_t bytes, void **out) {
    if (out == nullptr) return static_cast<int>(cudaErrorInvalidValue);
    *out = nullptr;
    return static_cast<int>(cudaHostAlloc(out, bytes, cudaHostAllocMapped | cudaHostAllocPortable));
}

int synth_host_free(void *p) { return static_cast<int>(cudaFreeHost(p)); }

}  // extern "C"

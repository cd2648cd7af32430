// synth_fill.cu -- libmoe_synth: device-side generator of synthetic expert
// objects, bit-identical to fp4_routed_expert_router_b200/synth.py.
//
// It holds none of the layer's arithmetic: it only writes uniform bytes
// (FP4 codes) and uniform exponents in [lo, hi] (UE8M0 scales) into one
// expert object in checkpoint layout (w1, w3, w2 codes, then s1, s3, s2
// scales; 10100.com article 151357339, sections "moe专家的容量瓶颈" and
// "SSD读取性能").  The generator is splitmix64 in counter mode (Steele, Lea,
// Flood, OOPSLA 2014): output i of the stream with key K is
// mix(K + (i+1) * 0x9E3779B97F4A7C15), so any slice of any tensor can be
// produced independently on the device or on the host.
#include <cuda_runtime.h>
#include <cstdint>

namespace {

constexpr uint64_t kGolden = 0x9E3779B97F4A7C15ull;

__host__ __device__ inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

uint64_t stream_key(uint64_t seed, int layer, int expert, int tensor) {
    const uint64_t sid = (static_cast<uint64_t>(layer & 0xFFFF) << 20) |
                         (static_cast<uint64_t>(expert & 0xFFFF) << 4) | static_cast<uint64_t>(tensor & 0xF);
    return mix64(mix64(seed) + (sid + 1) * kGolden);
}

struct Part {
    uint64_t key;
    uint64_t off;    // byte offset in the object
    uint64_t n;      // bytes
    int is_scale;
};

struct Parts {
    Part p[6];
    int lo, span;
};

__global__ void fill_kernel(uint8_t* dst, Parts ps) {
    const int which = blockIdx.y;
    const Part pt = ps.p[which];
    if (!pt.is_scale) {
        const uint64_t nw = pt.n / 8;
        for (uint64_t i = blockIdx.x * static_cast<uint64_t>(blockDim.x) + threadIdx.x; i < nw;
             i += static_cast<uint64_t>(gridDim.x) * blockDim.x) {
            const uint64_t z = mix64(pt.key + (i + 1) * kGolden);
            reinterpret_cast<uint64_t*>(dst + pt.off)[i] = z;
        }
    } else {
        for (uint64_t i = blockIdx.x * static_cast<uint64_t>(blockDim.x) + threadIdx.x; i < pt.n;
             i += static_cast<uint64_t>(gridDim.x) * blockDim.x) {
            const uint64_t z = mix64(pt.key + (i + 1) * kGolden);
            const uint64_t e = ((z >> 32) * static_cast<uint64_t>(ps.span)) >> 32;
            dst[pt.off + i] = static_cast<uint8_t>(ps.lo + e);
        }
    }
}

// Drop the L2 lines of a buffer without writing them back (its contents are
// garbage): one 128-byte line per thread.
__global__ void l2_discard_kernel(uint8_t* p, size_t lines) {
    for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < lines;
         i += static_cast<size_t>(gridDim.x) * blockDim.x)
        asm volatile("discard.global.L2 [%0], 128;" ::"l"(p + 128 * i) : "memory");
}

}  // namespace

extern "C" {

// Benchmark helper: after a buffer larger than L2 has been written to push
// every earlier line out of L2, discard that buffer's lines (no write-back),
// so the next kernel starts with a cold and clean L2 instead of paying for
// the flush buffer's dirty lines.  p 128-byte aligned, bytes a multiple of
// 128.  Returns a cudaError_t value (0 = ok).
int moe_synth_l2_discard(void* p, size_t bytes, void* stream) {
    if (!p || (reinterpret_cast<uintptr_t>(p) & 127) || (bytes & 127)) return static_cast<int>(cudaErrorInvalidValue);
    l2_discard_kernel<<<1184, 256, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<uint8_t*>(p), bytes / 128);
    return static_cast<int>(cudaGetLastError());
}

// Bytes of one expert object (same as moe_fp4_slot_bytes for a valid shape).
size_t moe_synth_expert_bytes(int hidden, int inter) {
    const size_t H = hidden, I = inter;
    return 2 * (I * H / 2 + I * H / 32) + (H * I / 2 + H * I / 32);
}

// Fill `dst` (device, moe_synth_expert_bytes bytes, 8-byte aligned) with the
// synthetic expert (seed, layer, expert).  hidden and inter must be multiples
// of 32 with I*H/2 a multiple of 8.  Returns a cudaError_t value (0 = ok).
int moe_synth_fill_expert(uint8_t* dst, uint64_t seed, int layer, int expert, int hidden, int inter,
                          int scale_lo, int scale_hi, void* stream) {
    if (!dst || hidden <= 0 || inter <= 0 || hidden % 32 || inter % 32 || scale_hi < scale_lo ||
        scale_lo < 0 || scale_hi > 255 || (reinterpret_cast<uintptr_t>(dst) & 7))
        return static_cast<int>(cudaErrorInvalidValue);
    const uint64_t H = hidden, I = inter;
    const uint64_t c13 = I * H / 2, c2 = H * I / 2, s13 = I * H / 32, s2 = H * I / 32;
    if (c13 % 8 || c2 % 8) return static_cast<int>(cudaErrorInvalidValue);
    Parts ps;
    // tensor ids as in synth.py: w1 0, s1 1, w3 2, s3 3, w2 4, s2 5
    ps.p[0] = {stream_key(seed, layer, expert, 0), 0, c13, 0};
    ps.p[1] = {stream_key(seed, layer, expert, 2), c13, c13, 0};
    ps.p[2] = {stream_key(seed, layer, expert, 4), 2 * c13, c2, 0};
    ps.p[3] = {stream_key(seed, layer, expert, 1), 2 * c13 + c2, s13, 1};
    ps.p[4] = {stream_key(seed, layer, expert, 3), 2 * c13 + c2 + s13, s13, 1};
    ps.p[5] = {stream_key(seed, layer, expert, 5), 2 * c13 + c2 + 2 * s13, s2, 1};
    ps.lo = scale_lo;
    ps.span = scale_hi - scale_lo + 1;
    fill_kernel<<<dim3(148, 6), 256, 0, static_cast<cudaStream_t>(stream)>>>(dst, ps);
    return static_cast<int>(cudaGetLastError());
}

}  // extern "C"

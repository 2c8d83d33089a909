// synth_fill.cu -- libmoe_synth.so: the seeded synthetic expert bytes, drawn on the GPU.
//
// Input generation only (no step of the MoE layer).  It draws the same bytes as the host
// generator in expert_ffn_token_b200/synth.py, from the same counter-based definition
// (SplitMix64's mixing function, Steele, Lea & Flood, OOPSLA 2014):
//   word(k, n) = mix64(k + (n + 1) * 0x9E3779B97F4A7C15)
//   raw byte p of a tensor  = byte p % 8 of word(k_raw, p / 8)
//   block i's d (and dmin)  = fp16(fp32(1e-3 + 9e-3 * (word(k_d, i) >> 11) * 2^-53))
//   Q5_1 block i's offset m = -16 * its dmin draw (exact in fp16)
// K-quant blocks that end past the row's logical width get scale and min 0 for the sub-blocks
// past it; pad bytes after a row's last block are 0.  The per-tensor keys are computed on the
// host and passed in.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

extern "C" {
typedef struct {
    uint64_t dst_off;       // byte offset of the tensor in the destination buffer
    uint64_t key_raw, key_d, key_dmin;
    int32_t rows, stride;   // row count, row stride in bytes (multiple of 16)
    int32_t nblocks;        // blocks per row
    int32_t block_bytes;    // 144, 176, 34 or 24
    int32_t kquant;         // 1: d and dmin at bytes 0-3 and packed scales at 4-15; 0: Q8_0;
                            // 2: Q5_1 (d and m = -16 * dmin draw at bytes 0-3)
    int32_t valid_last;     // sub-blocks of the last block inside the logical width (8 = all)
} synth_tensor;
}

namespace {

__device__ __forceinline__ uint64_t mix64(uint64_t z) {
    z ^= z >> 30;
    z *= 0xBF58476D1CE4E5B9ull;
    z ^= z >> 27;
    z *= 0x94D049BB133111EBull;
    z ^= z >> 31;
    return z;
}

__device__ __forceinline__ uint64_t word(uint64_t k, uint64_t n) {
    return mix64(k + (n + 1) * 0x9E3779B97F4A7C15ull);
}

__device__ __forceinline__ uint32_t scale_half(uint64_t w) {
    const double u = (double)(w >> 11) * 0x1.0p-53;
    const double v = __dadd_rn(1e-3, __dmul_rn(9e-3, u));
    return __half_as_ushort(__float2half_rn(__double2float_rn(v)));
}

// Scale/min byte `o` (4..15) of a K-quant block with only `valid` leading sub-blocks kept.
__device__ __forceinline__ uint32_t kill_scale_byte(uint32_t b, int o, int valid) {
    const int i = o - 4;                       // index into the 12 packed bytes
    for (int j = valid; j < 8; j++) {
        if (j < 4) {
            if (i == j || i == j + 4) b &= 0xC0u;
        } else {
            if (i == j + 4) b = 0;
            if (i == j - 4 || i == j) b &= 0x3Fu;
        }
    }
    return b;
}

__global__ void k_synth_fill(uint8_t *dst, const synth_tensor *tensors) {
    const synth_tensor T = tensors[blockIdx.y];
    const uint64_t nwords = (uint64_t)T.rows * T.stride / 8;
    const int packed = T.nblocks * T.block_bytes;
    for (uint64_t wi = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; wi < nwords;
         wi += (uint64_t)gridDim.x * blockDim.x) {
        const uint64_t p = wi * 8;
        const uint64_t row = p / T.stride;
        const int col0 = (int)(p % T.stride);
        const uint64_t raw = word(T.key_raw, wi);
        uint64_t outw = 0;
        for (int b = 0; b < 8; b++) {
            const int col = col0 + b;
            uint32_t v = (uint32_t)(raw >> (8 * b)) & 0xFFu;
            if (col >= packed) {
                v = 0;
            } else {
                const int blk = col / T.block_bytes, o = col % T.block_bytes;
                const uint64_t i = row * T.nblocks + blk;
                if (o < 2) {
                    v = (scale_half(word(T.key_d, i)) >> (8 * o)) & 0xFFu;
                } else if (T.kquant == 2 && o < 4) {
                    const uint32_t m = (scale_half(word(T.key_dmin, i)) + (4u << 10)) | 0x8000u;
                    v = (m >> (8 * (o - 2))) & 0xFFu;
                } else if (T.kquant == 1 && o < 4) {
                    v = (scale_half(word(T.key_dmin, i)) >> (8 * (o - 2))) & 0xFFu;
                } else if (T.kquant == 1 && o < 16 && blk == T.nblocks - 1 && T.valid_last < 8) {
                    v = kill_scale_byte(v, o, T.valid_last);
                }
            }
            outw |= (uint64_t)v << (8 * b);
        }
        *reinterpret_cast<uint64_t *>(dst + T.dst_off + p) = outw;
    }
}

}  // namespace

extern "C" int synth_fill_tensors(void *d_dst, const synth_tensor *host_tensors, int n,
                                  void *stream) {
    if (!d_dst || !host_tensors || n <= 0 || n > 65535) return 1;
    cudaStream_t st = (cudaStream_t)stream;
    synth_tensor *d_t = nullptr;
    if (cudaMallocAsync(&d_t, sizeof(synth_tensor) * n, st) != cudaSuccess) return 2;
    if (cudaMemcpyAsync(d_t, host_tensors, sizeof(synth_tensor) * n, cudaMemcpyHostToDevice, st) !=
        cudaSuccess)
        return 3;
    dim3 grid(148 * 4 / (n < 64 ? 1 : 8) + 1, n);
    k_synth_fill<<<grid, 256, 0, st>>>(static_cast<uint8_t *>(d_dst), d_t);
    if (cudaGetLastError() != cudaSuccess) return 4;
    if (cudaFreeAsync(d_t, st) != cudaSuccess) return 5;
    return 0;
}

// Internal declarations of libecco_b200: device-side table layout, kernel
// launchers and small device helpers shared by the kernels.
//
// Format: "Ecco: Improving Memory Bandwidth and Capacity for LLMs via
// Entropy-aware Cache Compression" (review page: "What carries the argument",
// Fig. 4 caption, free parameters).  The bit layout is documented in
// include/ecco.h.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "../../include/ecco.h"

namespace ecco {

constexpr int kG = 128;           // values per group
constexpr int kGAct = 64;         // values per group, activation format (2x)
constexpr int kNPat = 64;         // shared patterns per tensor
constexpr int kNCent = 15;        // centroids per pattern
constexpr int kNBook = 4;         // codebooks per pattern
constexpr int kNSym = 16;         // symbols (15 centroids + scale element)
constexpr int kLMax = 8;          // longest codeword
constexpr int kBlockBits = 512;
constexpr int kHdrBits = 16;
constexpr int kPayloadBits = 496;
constexpr int kRecBits = 15;
constexpr int kMaxRec = 16;

// Device-resident tables derived once from a blob (ecco_tables_create).
// Every array a kernel stages into shared memory is 16-byte aligned and a
// multiple of 16 bytes.
struct DevTables {
    float S_t;
    uint32_t pad0[3];
    float T16[kNPat][16];           // thresholds (C[j]+C[j+1])*0.5; [14], [15] = +inf
    float Ct[16][kNPat];            // centroid j of pattern p; row 15 = 1.0 (scale element)
    float2 ends[kNPat];             // (C[p][0], C[p][14])
    uint32_t lens4[kNPat][16];      // byte h = length of symbol s in codebook h
    uint32_t code[kNPat][kNBook][16];  // bits 0-7 codeword in stream order, bits 8-11 length
    // [t = h * 64 + p] (= header bits 8-15): the next 8 stream bits e -> symbol | length << 4, entry e at
    // byte e ^ ((t & 31) << 2) (word-level swizzle against bank conflicts, see lut_key)
    uint8_t lut[kNBook * kNPat][256];
    // Scale tables, filled on the device at creation with the same operations
    // the encoder would otherwise run per group (IEEE divide, E4M3 rounding,
    // fp32 multiply, correctly rounded reciprocal):
    float s_of_code[256];           // S_t * fp8(code); 0 for zero and NaN codes
    float inv_of_code[256];         // 1 / s_of_code (0 where s is 0)
    uint8_t code_of_mag[32768];     // E4M3(|x| / S_t), saturating, for every bf16 magnitude |x|
    float o_of_q[256];              // outlier record value q / 127 (IEEE divide) for each 8-bit code of q
    // Bucket map of the encoder's threshold search (threshold_bucket), filled
    // on the device at creation: per pattern (a, b, 1 if two thresholds share
    // a bucket, 0) and, per bucket n, the number of thresholds whose bucket is
    // below n.
    float4 qmap[kNPat];
    uint8_t qlo[kNPat][256];
};

}  // namespace ecco

struct ecco_tables {
    int device;
    ecco::DevTables* d;
};

namespace ecco {

// ------------------------------------------------------------ launchers

cudaError_t launch_encode(const ecco_tables* t, const uint16_t* x, const ecco_desc& d,
                          uint8_t* blocks, ecco_stats* stats, cudaStream_t s,
                          int select = ECCO_SELECT_MINMAX, int npat = kNPat);
cudaError_t launch_decode(const ecco_tables* t, const uint8_t* blocks, const ecco_desc& d,
                          uint16_t* y, cudaStream_t s);
cudaError_t launch_decode_spec(const ecco_tables* t, const uint8_t* blocks, const ecco_desc& d,
                               uint16_t* y, cudaStream_t s);
cudaError_t launch_gemv(const ecco_tables* t, const uint8_t* blocks, int64_t rows, int64_t cols,
                        const uint16_t* x, int batch, float* y, cudaStream_t s);
cudaError_t launch_gemm_tc(const ecco_tables* t, const uint8_t* blocks, int64_t rows, int64_t cols,
                           const uint16_t* x, int batch, float* y, cudaStream_t s);
cudaError_t launch_decode_multi(const ecco_segment* segs, int n, cudaStream_t s);
// Timeouts of the tensor-core pipeline's bounded waits: a host-visible flag
// (mapped pinned memory, allocated once) that a wait which gave up raises.
int* timeout_flag();
bool timeout_raised();
cudaError_t launch_wait_timeout_selftest(cudaStream_t s);
// Activation format: 64-value groups (the descriptor counts 64-value groups).
cudaError_t launch_encode_act(const ecco_tables* t, const uint16_t* x, const ecco_desc& d,
                              uint8_t* blocks, ecco_stats* stats, cudaStream_t s);
cudaError_t launch_decode_act(const ecco_tables* t, const uint8_t* blocks, const ecco_desc& d,
                              uint16_t* y, cudaStream_t s);
cudaError_t launch_encode_multi(const ecco_segment* segs, int n, ecco_stats* stats,
                                cudaStream_t s);

// Attention over a compressed KV cache: splits of 512 tokens (the fused
// kernel), then a merge.
int attention_splits(int seq_len);
cudaError_t launch_attention(const ecco_tables* kt, const ecco_tables* vt, const uint8_t* kblk,
                             const uint8_t* vblk, int64_t s_cap, int B, int H, int G, int S,
                             const uint16_t* q, float scale, float* out, float* ws, cudaStream_t s);
// Staged attention: chunks of staged_chunk_tokens() tokens decoded into
// `scratch` ([2][B*H][chunk][128] bf16) by the block decoder, then a split
// kernel without tables copies whole decoded rows into shared memory
// (cp.async) and runs the same products and softmax as launch_attention's
// kernel.  On B200 it is the faster of the two: the fused kernel's tables,
// stream words and tiles leave it half the decoder's resident warps, so its
// serial walk shows through.
int64_t staged_chunk_tokens(int B, int H, int seq_len);
// Splits of the staged path's kernel (256 tokens each): its partials hold
// 130 floats per (batch, query head, split).
int attention_staged_splits(int seq_len);
cudaError_t launch_attention_staged(const ecco_tables* kt, const ecco_tables* vt, const uint8_t* kblk,
                                    const uint8_t* vblk, int64_t s_cap, int B, int H, int G, int S,
                                    const uint16_t* q, float scale, float* out, float* ws, uint16_t* scratch,
                                    cudaStream_t s);

// Table learner (offline): the blob of one tensor from a device bf16 sample.
cudaError_t learn_tables(const uint16_t* x, int64_t n_groups, int G, int npat, uint64_t seed, uint8_t* blob,
                         cudaStream_t s);
int huffman_lengths(const double* w, int n, int max_len, uint8_t* lens);

int device_sm_count();

// Argument checks of the attention entry points (tables, sizes, pointers,
// alignment of blocks, q and out); ECCO_OK or the error code to return.
int check_attention(const ecco_tables* kt, const ecco_tables* vt, const uint8_t* kblk, const uint8_t* vblk,
                    int64_t s_cap, int batch, int kv_heads, int group, int seq_len, const uint16_t* q,
                    const float* out);

// Devices a per-kernel "already configured" bit set can name; a device index
// at or beyond it is configured on every launch (correct, just slower).
constexpr int kMaxDeviceBits = 64;

// Raises `fn`'s dynamic shared-memory limit to `bytes` on the current device,
// once per device: `done` holds one bit per device whose call succeeded.
// Safe to call from several host threads at once (a race only repeats the
// idempotent attribute call).
inline cudaError_t set_max_smem_once(std::atomic<uint64_t>& done, const void* fn, size_t bytes)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = (dev >= 0 && dev < kMaxDeviceBits) ? (1ull << dev) : 0ull;
    if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
    return e;
}

// ------------------------------------------------------------ device helpers
__device__ __forceinline__ float bf16_bits_to_f32(uint32_t h) { return __uint_as_float(h << 16); }

__device__ __forceinline__ uint32_t f32_to_bf16_bits(float f)
{
    return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(f));
}

__device__ __forceinline__ float e4m3_to_f32(uint32_t code)
{
    __half_raw hr = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)code, __NV_E4M3);
    return __half2float(__half(hr));
}

// Scale codes whose E4M3 value is zero or NaN mark an all-zero block.
__device__ __forceinline__ bool scale_code_is_null(uint32_t code)
{
    uint32_t mag = code & 0x7fu;
    return mag == 0u || mag == 0x7fu;
}

// 32 bytes from global memory through the read-only path (one 256-bit load;
// p 32-byte aligned).
__device__ __forceinline__ void ldg_nc_v8(const void* p, uint4& a, uint4& b)
{
    asm volatile("ld.global.nc.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(a.x), "=r"(a.y), "=r"(a.z), "=r"(a.w), "=r"(b.x), "=r"(b.y), "=r"(b.z), "=r"(b.w)
                 : "l"(p));
}

__device__ __forceinline__ uint4 ldg_nc_v4(const void* p)
{
    uint4 r;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ float warp_min_f32(float v)
{
    float r;
    asm volatile("redux.sync.min.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
    return r;
}

__device__ __forceinline__ float warp_max_f32(float v)
{
    float r;
    asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
    return r;
}

}  // namespace ecco

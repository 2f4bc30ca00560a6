// Fused decode + batched matrix-vector product on the 5th-generation tensor
// cores (tcgen05), for batch 5..16.
//
// y[b][r] = sum_k W~[r][k] x[b][k]: with a batch of activations the product
// is a real dense contraction (M = rows, N = batch, K = cols), so the decoded
// weights go to the tensor cores instead of 16 FMAs per weight on CUDA cores.
// (Review page, figure list: "Normalized Memory Requests for a GEMM Kernel" --
// only compressed weights cross the memory bus.)
//
// CTA = 512 threads = 4 M-tiles of 128 rows; the CTA walks a range of column
// groups, every thread decoding its own row's block (the block walker of
// ecco_block.cuh).  Each 16 decoded values of a row (one K = 16 slice) go into
// that tile's A buffer in shared memory (K-major, no swizzle: 8-row x 16-byte
// core matrices); when the tile's 128 threads have written a slice, one
// elected thread issues tcgen05.mma (M = 128, N = 16, K = 16, bf16 in, fp32
// accumulate in tensor memory) and commits it to the buffer's mbarrier; the
// buffer is written again only after that MMA completed.  A is double
// buffered, so decoding the next slice overlaps the MMA of the current one.
// x for the CTA's whole column range is staged once as the B operand.
//
// Outlier records are known only at the end of a block's stream, after its
// slices went to the tensor cores, so their effect is added on CUDA cores as
// (new - old) * x.  Partial sums of column ranges are combined with fp32
// atomics, as in the CUDA-core kernel.
//
// Every wait on an mbarrier is bounded; a wait that gives up increments a
// device counter (ecco_device_timeouts) and the kernel finishes without
// touching the buffer again.
#include "ecco_block.cuh"

namespace ecco {

__device__ unsigned int g_timeouts = 0;

namespace {

constexpr int kTcThreads = 512;
constexpr int kTcTiles = kTcThreads / 128;
constexpr int kTcStride = kTcThreads;        // word staging column stride
constexpr int kSliceBytes = 128 * 16 * 2;    // one 128 x 16 bf16 A slice
constexpr int kBSliceBytes = 16 * 16 * 2;    // one 16 x 16 bf16 B slice
constexpr int kMaxGroups = 8;                // column groups per CTA (x staged for all)
constexpr uint32_t kSpinLimit = 1u << 22;  // polls; with the back-off below, well under a second

constexpr size_t kOffLut = 0;
constexpr size_t kOffCt = kOffLut + 65536;
constexpr size_t kOffWords = kOffCt + 4096;
constexpr size_t kOffNib = kOffWords + 16 * kTcStride * 4;
constexpr size_t kOffA = kOffNib + 16 * kTcThreads * 4;
constexpr size_t kOffB = kOffA + (size_t)kTcTiles * 2 * kSliceBytes;
constexpr size_t kOffBar = kOffB + (size_t)kMaxGroups * 8 * kBSliceBytes;
constexpr size_t kTcSmem = kOffBar + 128 + kSmemAlign;

// Instruction descriptor: D fp32 (bits 4-5 = 1), A and B bf16 (bits 7-9, 10-12
// = 1), both K-major, N >> 3 in bits 17-22, M >> 4 in bits 24-28.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((16u >> 3) << 17) | ((128u >> 4) << 24);

// Shared-memory matrix descriptor, K-major without swizzle: start >> 4,
// leading byte offset (between the two 8-element K halves) 128 B, stride byte
// offset (between 8-row groups) 256 B, descriptor version 1.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr)
{
    return (uint64_t)((addr >> 4) & 0x3fffu) | ((uint64_t)(128u >> 4) << 16) | ((uint64_t)(256u >> 4) << 32) |
           (1ull << 46);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p)
{
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

// Waits for the phase with the given parity to complete: non-blocking polls,
// with a short sleep after the first few, at most kSpinLimit of them.
// Returns false (and counts a timeout) if it gave up.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity)
{
    const uint32_t a = smem_u32(bar);
    for (uint32_t i = 0; i < kSpinLimit; ++i) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(a), "r"(parity)
            : "memory");
        if (done) return true;
        if (i >= 16) __nanosleep(64);
    }
    atomicAdd(&g_timeouts, 1u);
    return false;
}

__device__ __forceinline__ void named_sync(int id, int n)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(kIdesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t* bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// Byte offset of element (row, k) inside a 128 x 16 K-major slice.
__device__ __forceinline__ uint32_t a_offset(int row, int khalf)
{
    return (uint32_t)((row >> 3) * 256 + khalf * 128 + (row & 7) * 16);
}

__global__ void __launch_bounds__(kTcThreads, 1)
    gemm_tc_kernel(const DevTables* __restrict__ tb, const uint8_t* __restrict__ blocks, int64_t rows,
                   int64_t gpr, const uint16_t* __restrict__ x, int batch, int64_t cols, int splits,
                   float* __restrict__ y)
{
    extern __shared__ __align__(128) uint8_t smem_raw[];
    uint8_t* smem = aligned_smem(smem_raw);
    uint8_t* s_lut = smem + kOffLut;
    float* s_Ct = reinterpret_cast<float*>(smem + kOffCt);
    uint32_t* s_w = reinterpret_cast<uint32_t*>(smem + kOffWords);
    uint32_t* s_nib = reinterpret_cast<uint32_t*>(smem + kOffNib);
    uint8_t* s_A = smem + kOffA;
    uint8_t* s_B = smem + kOffB;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);  // [tile][2] then done[tile]
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + kOffBar + 96);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int tile = warp >> 2;             // 4 warps per 128-row tile
    const int trow = (warp & 3) * 32 + lane;  // row inside the tile = TMEM lane

    // this CTA's column groups
    const int64_t g_begin = gpr * blockIdx.y / splits, g_end = gpr * (blockIdx.y + 1) / splits;
    const int ng = (int)(g_end - g_begin);

    stage_tables<kTcThreads>(tb, s_lut, s_Ct, tid);
    // B: x[b][k] for the column range, as ng * 8 slices of 16 x 16, K-major
    for (int e = tid; e < ng * 128 * 16; e += kTcThreads) {
        const int b = e & 15, k = e >> 4;  // k within the range
        uint16_t v = 0;
        if (b < batch) v = x[(int64_t)b * cols + g_begin * kG + k];
        const int slice = k >> 4, kk = k & 15;
        const uint32_t off = slice * kBSliceBytes + (b >> 3) * 256 + (kk >> 3) * 128 + (b & 7) * 16 + (kk & 7) * 2;
        *reinterpret_cast<uint16_t*>(s_B + off) = v;
    }
    if (tid == 0) {
        for (int i = 0; i < 3 * kTcTiles; ++i) mbar_init(&bars[i], 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(s_tmem)),
                     "r"(64)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // B staged by generic stores
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem_d = *s_tmem + (uint32_t)(16 * tile);  // this tile's 16 fp32 columns
    const float S_t = tb->S_t;

    const int64_t row = (int64_t)blockIdx.x * kTcThreads + tile * 128 + trow;
    const bool row_ok = row < rows;
    uint32_t* ws = s_w + tid;
    uint32_t* nibs = s_nib + tid;
    uint8_t* A0 = s_A + tile * 2 * kSliceBytes;
    const bool issuer = (warp & 3) == 0 && lane == 0;
    uint64_t* bar_buf = &bars[tile * 2];
    uint64_t* bar_done = &bars[2 * kTcTiles + tile];
    float corr[16];
#pragma unroll
    for (int b = 0; b < 16; ++b) corr[b] = 0.0f;
    bool ok = true;
    int t = 0;  // slice counter over the CTA's column range

    for (int gi = 0; gi < ng; ++gi) {
        uint4 q0 = make_uint4(0, 0, 0, 0), q1 = q0, q2 = q0, q3 = q0;
        if (row_ok) {
            const uint8_t* src = blocks + (row * gpr + g_begin + gi) * ECCO_BLOCK_BYTES;
            q0 = ldg_nc_v4(src);
            q1 = ldg_nc_v4(src + 16);
            q2 = ldg_nc_v4(src + 32);
            q3 = ldg_nc_v4(src + 48);
        }
        const uint32_t code = q0.x & 0xffu;
        const int p = (int)((q0.x >> 8) & 63u);
        const float s = (row_ok && !scale_code_is_null(code)) ? __fmul_rn(S_t, e4m3_to_f32(code)) : 0.0f;
        stage_words(ws, kTcStride, q0, q1, q2, q3);
        const ValuePlanes vp = make_planes(s, s_Ct, p);
        const uint8_t* lut = s_lut + ((q0.x >> 8) & 255u) * 256;
        Stream st{q0.x, q0.y, kHdrBits, 2, kPayloadBits};

#pragma unroll 1
        for (int sl = 0; sl < 8; ++sl, ++t) {
            uint32_t wa[4], wb[4];
            nibs[(2 * sl) * kTcThreads] = chunk_values(st, lut, ws, kTcStride, vp, wa);
            nibs[(2 * sl + 1) * kTcThreads] = chunk_values(st, lut, ws, kTcStride, vp, wb);
            const int buf = t & 1, use = t >> 1;
            if (use >= 1 && ok) ok = mbar_wait(&bar_buf[buf], (uint32_t)((use - 1) & 1));
            uint8_t* A = A0 + buf * kSliceBytes;
            if (ok) {
                *reinterpret_cast<uint4*>(A + a_offset(trow, 0)) = make_uint4(wa[0], wa[1], wa[2], wa[3]);
                *reinterpret_cast<uint4*>(A + a_offset(trow, 1)) = make_uint4(wb[0], wb[1], wb[2], wb[3]);
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            named_sync(1 + tile, 128);
            if (issuer && ok) {
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                const uint64_t ad = smem_desc(smem_u32(A));
                const uint64_t bd = smem_desc(smem_u32(s_B + (gi * 8 + sl) * kBSliceBytes));
                mma_bf16(tmem_d, ad, bd, t > 0 ? 1u : 0u);
                mma_commit(&bar_buf[buf]);
            }
        }

        if (s != 0.0f && st.room >= 0) {  // outlier records: add (new - old) * x
            const int n = min(kMaxRec, st.room / kRecBits);
            const int at0 = kBlockBits - st.room;
            // Newest first: the last record of an element wins, so an element
            // already seen (128-bit mask) is skipped.
            uint32_t seen0 = 0u, seen1 = 0u, seen2 = 0u, seen3 = 0u;
            for (int k = n - 1; k >= 0; --k) {
                uint32_t rec = read_record(ws, kTcStride, at0 + k * kRecBits);
                int i = (int)(rec & 127u);
                const uint32_t bit = 1u << (i & 31), q = (uint32_t)i >> 5;
                const uint32_t was = (q == 0u ? seen0 : q == 1u ? seen1 : q == 2u ? seen2 : seen3) & bit;
                seen0 |= (q == 0u) ? bit : 0u;
                seen1 |= (q == 1u) ? bit : 0u;
                seen2 |= (q == 2u) ? bit : 0u;
                seen3 |= (q == 3u) ? bit : 0u;
                if (was) continue;
                float nv = bf16_bits_to_f32(f32_to_bf16_bits(__fmul_rn(s, __ldg(&tb->o_of_q[rec >> 7]))));
                uint32_t osym = (nibs[(i >> 3) * kTcThreads] >> (4 * (i & 7))) & 15u;
                uint32_t ow = (osym < 8) ? ((osym < 4) ? vp.lo[0] : vp.lo[1]) : ((osym < 12) ? vp.lo[2] : vp.lo[3]);
                uint32_t oh = (osym < 8) ? ((osym < 4) ? vp.hi[0] : vp.hi[1]) : ((osym < 12) ? vp.hi[2] : vp.hi[3]);
                uint32_t sh = 8 * (osym & 3);
                float ov = __uint_as_float((((ow >> sh) & 0xffu) | (((oh >> sh) & 0xffu) << 8)) << 16);
                float dv = nv - ov;
                const int sl = i >> 4, kk = i & 15;
                const uint8_t* Bs = s_B + (gi * 8 + sl) * kBSliceBytes + (kk >> 3) * 128 + (kk & 7) * 2;
#pragma unroll
                for (int b = 0; b < 16; ++b) {
                    float xv = bf16_bits_to_f32(*reinterpret_cast<const uint16_t*>(Bs + (b >> 3) * 256 + (b & 7) * 16));
                    corr[b] = fmaf(dv, xv, corr[b]);
                }
            }
        }
    }

    // all MMAs of this tile done -> read the accumulator rows
    if (issuer && ok) mma_commit(bar_done);
    if (ok && t > 0) ok = mbar_wait(bar_done, 0u);
    __syncwarp();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    uint32_t v[16];
    const uint32_t taddr = tmem_d + ((uint32_t)((warp & 3) * 32) << 16);
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
    if (row_ok && ok && t > 0) {
#pragma unroll
        for (int b = 0; b < 16; ++b)
            if (b < batch) atomicAdd(&y[(int64_t)b * rows + row], __uint_as_float(v[b]) + corr[b]);
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(*s_tmem), "r"(64) : "memory");
}

}  // namespace

size_t gemm_tc_smem() { return kTcSmem; }

cudaError_t launch_gemm_tc(const ecco_tables* t, const uint8_t* blocks, int64_t rows, int64_t cols,
                           const uint16_t* x, int batch, float* y, cudaStream_t s)
{
    static std::atomic<uint64_t> configured{0};
    if (cudaError_t e0 = set_max_smem_once(configured, (const void*)gemm_tc_kernel, kTcSmem); e0 != cudaSuccess)
        return e0;
    cudaError_t e = cudaMemsetAsync(y, 0, sizeof(float) * (size_t)batch * (size_t)rows, s);
    if (e != cudaSuccess) return e;
    const int64_t gpr = cols / kG;
    const int64_t chunks = (rows + kTcThreads - 1) / kTcThreads;
    int64_t splits = (int64_t)device_sm_count() / chunks;  // one wave of CTAs
    if (splits < (gpr + kMaxGroups - 1) / kMaxGroups) splits = (gpr + kMaxGroups - 1) / kMaxGroups;
    if (splits > gpr) splits = gpr;
    if (splits < 1) splits = 1;
    dim3 grid((unsigned)chunks, (unsigned)splits);
    gemm_tc_kernel<<<grid, kTcThreads, kTcSmem, s>>>(t->d, blocks, rows, gpr, x, batch, cols, (int)splits, y);
    return cudaGetLastError();
}

}  // namespace ecco

extern "C" int ecco_device_timeouts(unsigned int* out)
{
    if (!out) return ECCO_ERR_ARG;
    return cudaMemcpyFromSymbol(out, ecco::g_timeouts, sizeof(unsigned int)) == cudaSuccess ? ECCO_OK : ECCO_ERR_CUDA;
}

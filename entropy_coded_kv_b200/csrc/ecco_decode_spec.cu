// Speculative warp-parallel decoder: the review page's decompressor design
// (Fig. 8 caption; referee major comment 1: parallel sub-decoders that start
// on overlapping segments of the block at every candidate offset, merged in a
// tree) mapped onto a warp.  The bench and the parity tests run it beside the
// thread-per-block decoder of ecco_decode.cu; it produces the same bf16 bits.
//
// One warp decodes one block.  Lane L < 31 owns the 16 payload bits
// [16 + 16L, 32 + 16L) (lane 31 owns none).  A codeword is at most 8 bits, so
// the first codeword that starts inside lane L's segment starts at one of
// its first 8 bits, and which one depends on every codeword before it.  The
// lane therefore decodes at every bit position of its segment -- 16 table
// lookups, independent of one another -- and, walking the positions from the
// last to the first, finds for every entry offset e in 0..7 the offset at
// which the chain of codewords leaves the segment: a map f_L from 8 offsets to
// 8 offsets, kept as 8 bytes.  The maps compose with byte permutes (the
// composed map's byte i is g's byte f(i)); a 5-step shuffle scan composes
// f_L o ... o f_0 in every lane (the tree merge), and lane L's entry offset is
// the composition over lanes 0..L-1 applied to 0 (the payload starts at
// offset 0 of lane 0's segment).  Each lane then walks its segment from its
// entry offset with the lengths it already looked up (no further lookups),
// counts its codewords, places them with a shuffle scan of the counts and
// writes their values into the warp's 256-byte row in shared memory.  A
// codeword that would end past bit 512 stops the walk (clipping); fewer than
// 128 codewords in all leave the rest of the row +0 and no records.  Else the
// lane that holds codeword 127 knows where the codewords end; the records are
// read there by lanes 0..n-1 at once, the last record of an element wins
// (__match_any_sync), and the row leaves in one coalesced 256-byte store.
//
// Cost: every bit position of the payload is looked up (496 lookups per block
// against 128 for the serial walk; all 31 lanes read one 256-byte table, so a
// warp's lookups conflict less), and the position walk, the scan of the maps
// and the segment walks are integer work.  Measured on the KV cache's K
// (262,144 blocks): 818 warp instructions per block against 76 for the
// thread-per-block walk, integer pipe 81% busy, 6x its time.
#include "ecco_block.cuh"

namespace ecco {
namespace {

constexpr int kSpecWarps = 32;
constexpr int kSpecThreads = kSpecWarps * 32;
constexpr size_t kSpecOffRows = 65536 + 4096;                    // after the decode tables and centroids
constexpr size_t kSpecOffVals = kSpecOffRows + kSpecWarps * 256;  // a row of 128 bf16 per warp
constexpr size_t kSpecSmem = kSpecOffVals + kSpecWarps * 32 + kSmemAlign;  // 16 bf16 values per warp

struct SpecArgs {
    const DevTables* tb;
    const uint8_t* blocks;
    uint16_t* y;
    ecco_desc d;
    int64_t total;
};

// A prmt selector whose 4 nibbles are the low 3 bits of x's 4 bytes.
__device__ __forceinline__ uint32_t byte_sel(uint32_t x)
{
    return __byte_perm(x | (x >> 4), 0u, 0x0020u);
}

// Byte j (0..15) of the 128-bit value E.
__device__ __forceinline__ uint32_t byte16(const uint32_t (&E)[4], int j)
{
    const uint32_t w = (j < 8) ? ((j < 4) ? E[0] : E[1]) : ((j < 12) ? E[2] : E[3]);
    return (w >> (8 * (j & 3))) & 0xffu;
}

__device__ __forceinline__ const uint8_t* block_ptr(const SpecArgs& A, int64_t item)
{
    const int64_t gpr = A.d.groups_per_row;
    const int64_t r = item / gpr, g = item - r * gpr;
    return A.blocks + (A.d.src_offset + r * A.d.src_row_stride + g) * ECCO_BLOCK_BYTES;
}

__global__ void __launch_bounds__(kSpecThreads, 1) decode_spec_kernel(const __grid_constant__ SpecArgs A)
{
    extern __shared__ __align__(16) uint8_t smem_raw[];
    uint8_t* smem = aligned_smem(smem_raw);
    uint8_t* s_lut = smem;
    float* s_Ct = reinterpret_cast<float*>(smem + 65536);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint16_t* row = reinterpret_cast<uint16_t*>(smem + kSpecOffRows) + warp * kG;
    uint16_t* vals = reinterpret_cast<uint16_t*>(smem + kSpecOffVals) + warp * 16;
    stage_tables<kSpecThreads>(A.tb, s_lut, s_Ct, tid);
    const float S_t = A.tb->S_t;
    __syncthreads();

    constexpr uint32_t kAll = 0xffffffffu;
    const int sbit = 16 + 16 * lane;  // this lane's segment; lane 31 has none
    const int64_t nwarps = (int64_t)gridDim.x * kSpecWarps;
    const int64_t first = (int64_t)blockIdx.x * kSpecWarps + warp;

    // lanes 0..15 hold the block's 16 words; the next block's are loaded one
    // block ahead, and the one after is on its way to L2
    uint32_t wnext = 0u;
    if (first < A.total && lane < 16) wnext = __ldg(reinterpret_cast<const uint32_t*>(block_ptr(A, first)) + lane);
    for (int64_t item = first; item < A.total; item += nwarps) {
        const uint32_t w = wnext;
        const int64_t nx = item + nwarps;
        wnext = 0u;
        if (nx < A.total && lane < 16) wnext = __ldg(reinterpret_cast<const uint32_t*>(block_ptr(A, nx)) + lane);
        if (lane == 0 && nx + nwarps < A.total)
            asm volatile("prefetch.global.L2 [%0];" ::"l"(block_ptr(A, nx + nwarps)));

        const int64_t gpr = A.d.groups_per_row;
        const int64_t r = item / gpr, g = item - r * gpr;
        uint2* drow = reinterpret_cast<uint2*>(A.y + (A.d.dst_offset + r * A.d.dst_row_stride + g) * kG) + lane;
        const uint32_t hdr = __shfl_sync(kAll, w, 0);
        const uint32_t code = hdr & 0xffu;
        if (scale_code_is_null(code)) {  // the whole block decodes to +0
            *drow = make_uint2(0u, 0u);
            continue;
        }
        const int p = (int)((hdr >> 8) & 63u);
        const uint32_t lkey = lut_key(s_lut, (hdr >> 8) & 255u);
        const float s = __fmul_rn(S_t, e4m3_to_f32(code));
        __syncwarp();  // the previous block's row and values are no longer read
        if (lane < 16) vals[lane] = (uint16_t)f32_to_bf16_bits(__fmul_rn(s, s_Ct[lane * kNPat + p]));
        reinterpret_cast<uint2*>(row)[lane] = make_uint2(0u, 0u);

        // bits [sbit, sbit + 32) of the block; bits past 511 read as 0
        const int wi = sbit >> 5;
        const uint32_t lo = __shfl_sync(kAll, w, wi & 31), hi = __shfl_sync(kAll, w, (wi + 1) & 31);
        const uint32_t win = __funnelshift_r(lo, hi, (uint32_t)sbit & 31u);

        // ---- one lookup at every bit position of the segment
        uint32_t e[16];
#pragma unroll
        for (int j = 0; j < 16; ++j)
            asm volatile("ld.shared.u8 %0, [%1];" : "=r"(e[j]) : "r"(lkey ^ ((win >> j) & 0xffu)) : "memory");
        uint32_t E[4];  // byte j: the table entry at position j (symbol | length << 4)
#pragma unroll
        for (int q = 0; q < 4; ++q)
            E[q] = __byte_perm(__byte_perm(e[4 * q], e[4 * q + 1], 0x0040u), __byte_perm(e[4 * q + 2], e[4 * q + 3], 0x0040u),
                               0x5410u);

        // ---- exit offsets, last position first: a codeword at j of length l
        // leaves the segment at j + l - 16 if j + l >= 16, else the chain goes
        // on from position j + l.  W nibble k = exit from position j + 1 + k.
        uint32_t W = 0u, f_lo = 0u, f_hi = 0u;
#pragma unroll
        for (int j = 15; j >= 0; --j) {
            const uint32_t l = e[j] >> 4;
            uint32_t x;
            if (j == 15)
                x = l - 1u;  // every codeword at the last position leaves
            else if (j < 8)
                x = (W >> (4u * (l - 1u))) & 15u;  // j + l <= 15: never leaves
            else
                x = ((uint32_t)j + l >= 16u) ? (uint32_t)j + l - 16u : (W >> (4u * (l - 1u))) & 15u;
            W = (W << 4) | x;
            if (j < 4)
                f_lo |= x << (8 * j);
            else if (j < 8)
                f_hi |= x << (8 * (j - 4));
        }
        if (lane == 31) {  // no segment: the identity map
            f_lo = 0x03020100u;
            f_hi = 0x07060504u;
        }

        // ---- tree merge: F_L = f_L o ... o f_0 by a shuffle scan
#pragma unroll
        for (int dlt = 1; dlt < 32; dlt <<= 1) {
            const uint32_t g_lo = __shfl_up_sync(kAll, f_lo, dlt), g_hi = __shfl_up_sync(kAll, f_hi, dlt);
            if (lane >= dlt) {
                const uint32_t n_lo = __byte_perm(f_lo, f_hi, byte_sel(g_lo));
                const uint32_t n_hi = __byte_perm(f_lo, f_hi, byte_sel(g_hi));
                f_lo = n_lo;
                f_hi = n_hi;
            }
        }
        int ent = (int)__shfl_up_sync(kAll, f_lo & 7u, 1);
        if (lane == 0) ent = 0;
        if (lane == 31) ent = 16;

        // ---- this lane's codewords, stopping at one that would end past bit
        // 512: their symbols in nibbles of (sy_hi:sy_lo), the count
        int cnt = 0;
        uint32_t sy_lo = 0u, sy_hi = 0u;
        for (int j = ent; j < 16;) {
            const uint32_t ej = byte16(E, j);
            const int l = (int)(ej >> 4);
            if (sbit + j + l > kBlockBits) break;
            sy_hi = __funnelshift_r(sy_lo, sy_hi, 28);  // (hi:lo) <<= 4
            sy_lo = (sy_lo << 4) | (ej & 15u);
            j += l;
            ++cnt;
        }
        int start = cnt;  // inclusive scan, then exclusive
#pragma unroll
        for (int dlt = 1; dlt < 32; dlt <<= 1) {
            const int t = __shfl_up_sync(kAll, start, dlt);
            if (lane >= dlt) start += t;
        }
        const int total = __shfl_sync(kAll, start, 31);
        start -= cnt;

        __syncwarp();  // the row is cleared and the values are in place
        // the most recent codeword is in the lowest nibble: codeword k of cnt
        // sits at nibble cnt - 1 - k
        for (int k = 0; k < cnt && start + k < kG; ++k) {
            const int sh = 4 * (cnt - 1 - k);
            const uint32_t sy = ((sh < 32) ? (sy_lo >> sh) : (sy_hi >> (sh - 32))) & 15u;
            row[start + k] = vals[sy];
        }

        if (total >= kG) {  // unclipped: outlier records follow codeword 127
            // the lane that holds it walks to its end
            const bool holds = start <= kG - 1 && kG - 1 < start + cnt;
            int endpos = 0;
            if (holds) {
                int j = ent;
                for (int k = start; k < kG; ++k) j += (int)(byte16(E, j) >> 4);
                endpos = sbit + j;
            }
            const unsigned own = __ballot_sync(kAll, holds);
            const int at0 = __shfl_sync(kAll, endpos, __ffs((int)own) - 1);
            const int n = min(kMaxRec, (kBlockBits - at0) / kRecBits);
            const int at = at0 + kRecBits * lane;
            const int rw = (at >> 5) & 31;
            const uint32_t r0 = __shfl_sync(kAll, w, rw), r1 = __shfl_sync(kAll, w, (rw + 1) & 31);
            const uint32_t rec = __funnelshift_r(r0, r1, (uint32_t)at & 31u) & 0x7fffu;
            const bool mine = lane < n;
            const int i = (int)(rec & (uint32_t)(kG - 1));
            const unsigned same = __match_any_sync(kAll, mine ? i : kG + lane);
            __syncwarp();  // codeword values written
            if (mine && lane == 31 - __clz((int)same))  // the last record of element i
                row[i] = (uint16_t)f32_to_bf16_bits(__fmul_rn(s, q_over_127((int)(int8_t)(uint8_t)(rec >> 7))));
        }
        __syncwarp();
        *drow = reinterpret_cast<const uint2*>(row)[lane];
    }
}

}  // namespace

cudaError_t launch_decode_spec(const ecco_tables* t, const uint8_t* blocks, const ecco_desc& d, uint16_t* y,
                               cudaStream_t s)
{
    static std::atomic<uint64_t> configured{0};
    cudaError_t e = set_max_smem_once(configured, (const void*)decode_spec_kernel, kSpecSmem);
    if (e != cudaSuccess) return e;
    SpecArgs A;
    A.tb = t->d;
    A.blocks = blocks;
    A.y = y;
    A.d = d;
    A.total = d.rows * d.groups_per_row;
    const int64_t want = (A.total + kSpecWarps - 1) / kSpecWarps;
    const int64_t cap = device_sm_count();
    const int grid = (int)(want < cap ? want : cap);
    decode_spec_kernel<<<grid, kSpecThreads, kSpecSmem, s>>>(A);
    return cudaGetLastError();
}

}  // namespace ecco

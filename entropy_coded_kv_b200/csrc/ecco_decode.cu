// Decoder: one thread per 512-bit block.
//
// The review page's decompressor ("Ecco: Improving Memory Bandwidth and
// Capacity for LLMs via Entropy-aware Cache Compression", Fig. 8 caption and
// referee comment 1) is a 64-way hardware decoder that speculates at every bit
// offset to beat the serial dependency of one variable-length stream.  A
// B200 has millions of independent blocks in flight instead, so here every
// thread walks one block's stream serially and parallelism comes from the
// blocks: the serial chain (one shared-memory table lookup per symbol) is
// hidden by 28 resident warps per SM, and no work is spent on offsets that
// turn out to be wrong.  (ecco_decode_spec.cu builds the page's speculative
// scheme on a warp per block, for comparison: it is several times slower.)
//
// G = 64 is the activation format (64 values per 512-bit block, the review
// page's 2x ratio for activations); everything else is shared.  Activation
// blocks nearly always carry all 16 outlier records, so there the rows are
// assembled in shared memory (one 144-byte row per thread, 768 threads), the
// records patch the row there, and the row goes out with full 32-byte stores
// instead of 16 scattered 2-byte ones.
//
// Per block: parse the header (scale code, pattern, codebook), form the 16
// output values bf16(s * C[p][j]) as register byte planes, decode the stream
// 8 symbols at a time (ecco_block.cuh), write each 16 decoded values with one
// 32-byte store (lane pairs write 64 contiguous bytes of one row per
// instruction), then apply the outlier records of an unclipped stream.
#include <algorithm>

#include "ecco_block.cuh"

namespace ecco {
namespace {

constexpr size_t kDecSmemLut = sizeof(((DevTables*)0)->lut);  // 65536
constexpr size_t kDecSmemCt = sizeof(((DevTables*)0)->Ct);    // 4096
constexpr int kRowWords = 36;  // staged 64-value row: 32 words + 4 pad (16-byte stores conflict-free)

// Threads per CTA; word k of thread t's block at k * threads + t (conflict-free).
template <int G>
constexpr int dec_threads()
{
    return G == kG ? 896 : 768;  // 896: 72 registers for the paired stores below
}

template <int G>
constexpr size_t dec_smem()
{
    return kSmemAlign + kDecSmemLut + kDecSmemCt + (size_t)16 * dec_threads<G>() * 4 +
           (G == kG ? 0 : (size_t)dec_threads<G>() * kRowWords * 4);
}

// WIDE: blocks and output both 32-byte aligned: 32-byte block loads and
// stores (a 64-byte block in two loads: 2.7% faster on the long-context
// cache than four 16-byte loads); else 16-byte loads and stores.
template <bool WIDE>
__device__ __forceinline__ void store16(uint16_t* dst, const uint32_t a[4], const uint32_t b[4])
{
    if (WIDE) {
        stg256(dst, a, b);
    } else {
        *reinterpret_cast<uint4*>(dst) = make_uint4(a[0], a[1], a[2], a[3]);
        *reinterpret_cast<uint4*>(dst + 8) = make_uint4(b[0], b[1], b[2], b[3]);
    }
}

// One tensor's share of a launch: its tables, buffers, descriptor, and where
// its blocks start in the launch's concatenated block index.
struct DecSeg {
    const DevTables* tb;
    const uint8_t* src;
    uint16_t* dst;
    ecco_desc d;
    int64_t begin, count;
};

// Passed by value (a __grid_constant__ kernel parameter): no device-side
// segment table has to be allocated or copied.
template <int MAXSEG>
struct DecParams {
    int n_seg;
    int64_t total;
    DecSeg seg[MAXSEG];
};

// Each CTA decodes one contiguous, equal share of all blocks of the launch,
// segment by segment, restaging the segment's tables in shared memory when
// its share crosses into the next segment.
template <bool WIDE, int MAXSEG, int G>
__global__ void __launch_bounds__(dec_threads<G>(), 1) decode_kernel(const __grid_constant__ DecParams<MAXSEG> P)
{
    constexpr int kDecThreads = dec_threads<G>(), kWordStride = kDecThreads;
    constexpr bool kRows = G != kG;  // rows assembled in shared memory
    extern __shared__ __align__(16) uint8_t smem_raw[];
    uint8_t* smem = aligned_smem(smem_raw);
    uint8_t* s_lut = smem;
    float* s_Ct = reinterpret_cast<float*>(smem + kDecSmemLut);
    uint32_t* s_w = reinterpret_cast<uint32_t*>(smem + kDecSmemLut + kDecSmemCt);
    const int tid = threadIdx.x;
    uint32_t* ws = s_w + tid;
    uint32_t* row = s_w + 16 * kWordStride + tid * kRowWords;  // kRows only

    const int64_t share = (P.total + gridDim.x - 1) / gridDim.x;
    int64_t lo = (int64_t)blockIdx.x * share;
    const int64_t hi = min(P.total, lo + share);
    for (int si = 0; si < P.n_seg && lo < hi; ++si) {
        const DecSeg& S = P.seg[si];
        const int64_t seg_end = S.begin + S.count;
        if (seg_end <= lo) continue;
        const int64_t stop = min(hi, seg_end);
        const DevTables* tb = S.tb;
        __syncthreads();  // the previous segment's tables are no longer read
        stage_tables<kDecThreads>(tb, s_lut, s_Ct, tid);
        const float S_t = tb->S_t;
        __syncthreads();

        // local group index within the segment; consecutive threads take
        // consecutive groups.  The CTA's part of the segment is spread evenly
        // over the fewest rounds of at most kDecThreads (4 rounds of 886 rather
        // than 3 of 1024 and one of 470), so no round runs the SM half empty.
        // (32-bit: a segment holds fewer than 2^31 - 2048 groups, see check_desc)
        const int gpr = (int)S.d.groups_per_row;
        const int part = (int)(stop - lo);
        const int rounds = (part + kDecThreads - 1) / kDecThreads;
        const int per_round = (part + rounds - 1) / rounds;
        const int stride_r = per_round / gpr, stride_g = per_round % gpr;
        int item = (int)(lo - S.begin) + tid;
        const int end = (tid < per_round) ? (int)(stop - S.begin) : 0;
        int r = item / gpr, g = item - r * gpr;
        for (; item < end; item += per_round) {
            const uint8_t* src = S.src + (S.d.src_offset + (int64_t)r * S.d.src_row_stride + g) * ECCO_BLOCK_BYTES;
            uint16_t* dst = S.dst + (S.d.dst_offset + (int64_t)r * S.d.dst_row_stride + g) * G;
            g += stride_g;
            r += stride_r;
            if (g >= gpr) {
                g -= gpr;
                r += 1;
            }
            if (item + per_round < end)  // this thread's next block: on its way to L2 while this one decodes
                asm volatile("prefetch.global.L2 [%0];" ::"l"(S.src + (S.d.src_offset + (int64_t)r * S.d.src_row_stride + g) *
                                                                            ECCO_BLOCK_BYTES));

            uint4 q0, q1, q2, q3;
            if constexpr (WIDE) {
                ldg_nc_v8(src, q0, q1);
                ldg_nc_v8(src + 32, q2, q3);
            } else {
                q0 = ldg_nc_v4(src);
                q1 = ldg_nc_v4(src + 16);
                q2 = ldg_nc_v4(src + 32);
                q3 = ldg_nc_v4(src + 48);
            }
            const uint32_t code = q0.x & 0xffu;
            if (scale_code_is_null(code)) {
                const uint32_t z[4] = {0u, 0u, 0u, 0u};
#pragma unroll
                for (int k = 0; k < G / 16; ++k) store16<WIDE>(dst + 16 * k, z, z);
                continue;
            }
            stage_words(ws, kWordStride, q0, q1, q2, q3);
            const int p = (int)((q0.x >> 8) & 63u);
            const uint32_t lkey = lut_key(s_lut, (q0.x >> 8) & 255u);  // table h * 64 + p
            const float s = __fmul_rn(S_t, e4m3_to_f32(code));
            const ValuePlanes vp = make_planes(s, s_Ct, p);

            Stream st{q0.x, q0.y, kHdrBits, 2, kPayloadBits};
            // Lanes 2k and 2k+1 store 64 contiguous bytes of one row per
            // instruction (chunks c and c+1; each lane sends its partner the
            // chunk that belongs to the partner's store), so a warp store
            // touches 16 rows rather than 32: half the L1 wavefronts for the
            // row stores, 4% off the long-context decode.  It needs both lanes
            // of every pair on this block (not at a warp's ragged end or
            // beside a zero-scale block) and 32-byte aligned rows.
            const unsigned pm = __activemask();
            const bool pair_here = WIDE && !kRows && ((pm >> ((threadIdx.x & 31u) ^ 1u)) & 1u);
            uint16_t* pdst = reinterpret_cast<uint16_t*>(__shfl_xor_sync(pm, reinterpret_cast<uintptr_t>(dst), 1));
            if (__all_sync(pm, pair_here)) {
                const bool odd = threadIdx.x & 1u;
#pragma unroll 1
                for (int c = 0; c < G / 16; c += 2) {
                    uint32_t a0[4], b0[4], a1[4], b1[4], ra[4], rb[4];
                    chunk_values(st, lkey, ws, kWordStride, vp, a0);
                    chunk_values(st, lkey, ws, kWordStride, vp, b0);
                    chunk_values(st, lkey, ws, kWordStride, vp, a1);
                    chunk_values(st, lkey, ws, kWordStride, vp, b1);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {  // the even lane sends chunk c + 1, the odd lane chunk c
                        ra[k] = __shfl_xor_sync(pm, odd ? a0[k] : a1[k], 1);
                        rb[k] = __shfl_xor_sync(pm, odd ? b0[k] : b1[k], 1);
                    }
                    // the even lane's row, then the odd lane's
                    if (odd) store16<WIDE>(pdst + 16 * (c + 1), ra, rb); else store16<WIDE>(dst + 16 * c, a0, b0);
                    if (odd) store16<WIDE>(dst + 16 * (c + 1), a1, b1); else store16<WIDE>(pdst + 16 * c, ra, rb);
                }
            } else
#pragma unroll 1
            for (int c = 0; c < G / 16; ++c) {  // 16 symbols, one 32-byte store each
                uint32_t wa[4], wb[4];
                chunk_values(st, lkey, ws, kWordStride, vp, wa);
                chunk_values(st, lkey, ws, kWordStride, vp, wb);
                if constexpr (kRows) {
                    *reinterpret_cast<uint4*>(row + 8 * c) = make_uint4(wa[0], wa[1], wa[2], wa[3]);
                    *reinterpret_cast<uint4*>(row + 8 * c + 4) = make_uint4(wb[0], wb[1], wb[2], wb[3]);
                } else {
                    store16<WIDE>(dst + 16 * c, wa, wb);
                }
            }

            if (st.room >= 0) {  // unclipped: outlier records follow the codewords
                // Each record is read at its own offset (independent loads,
                // no chain through the stream window); q / 127 by one
                // correction step rather than a table gather, which would add
                // to the L1 traffic.
                const int n = min(kMaxRec, st.room / kRecBits);
                const int at0 = kBlockBits - st.room;
                for (int k = 0; k < n; ++k) {
                    const uint32_t rec = read_record(ws, kWordStride, at0 + k * kRecBits);
                    const int i = (int)(rec & (uint32_t)(G - 1));  // the 7-bit index, modulo G
                    const float o = q_over_127((int)(int8_t)(uint8_t)(rec >> 7));
                    const uint16_t v = (uint16_t)f32_to_bf16_bits(__fmul_rn(s, o));
                    if constexpr (kRows)
                        reinterpret_cast<uint16_t*>(row)[i] = v;
                    else
                        dst[i] = v;
                }
            }
            if constexpr (kRows) {
                // A warp whose 32 rows follow one another in the output (every
                // lane here, each row right after the previous lane's) writes
                // them as G/16 fully contiguous 1 KB stores: lane L stores bytes
                // 32 L .. 32 L + 31 of each, read from the staged row they
                // belong to, so an instruction touches 8 rows instead of 32.
                const unsigned am = __activemask();
                const int lane = tid & 31;
                const uintptr_t d0 = __shfl_sync(am, reinterpret_cast<uintptr_t>(dst), 0);
                const bool follows = reinterpret_cast<uintptr_t>(dst) == d0 + (uintptr_t)lane * G * 2;
                if (am == 0xffffffffu && __all_sync(am, follows)) {
                    __syncwarp();  // every lane's row, records included, is staged
                    const uint32_t* wrows = s_w + 16 * kWordStride + (tid & ~31) * kRowWords;
#pragma unroll
                    for (int c = 0; c < G / 16; ++c) {
                        const int k = 32 * c + lane;  // 32-byte piece k of the warp's rows
                        const uint32_t* src = wrows + (k / (G / 16)) * kRowWords + 8 * (k % (G / 16));
                        const uint4 a = *reinterpret_cast<const uint4*>(src);
                        const uint4 b = *reinterpret_cast<const uint4*>(src + 4);
                        const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
                        store16<WIDE>(reinterpret_cast<uint16_t*>(d0) + 16 * k, wa, wb);
                    }
                    __syncwarp();  // the rows are read before the lanes stage their next ones
                } else {
#pragma unroll
                    for (int c = 0; c < G / 16; ++c) {
                        const uint4 a = *reinterpret_cast<const uint4*>(row + 8 * c);
                        const uint4 b = *reinterpret_cast<const uint4*>(row + 8 * c + 4);
                        const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
                        store16<WIDE>(dst + 16 * c, wa, wb);
                    }
                }
            }
        }
        lo = stop;
    }
}

template <bool WIDE, int MAXSEG, int G = kG>
cudaError_t run_decode(const DecParams<MAXSEG>& P, cudaStream_t s)
{
    static std::atomic<uint64_t> configured{0};
    cudaError_t e = set_max_smem_once(configured, (const void*)decode_kernel<WIDE, MAXSEG, G>, dec_smem<G>());
    if (e != cudaSuccess) return e;
    // one resident CTA per SM; a small launch is spread over the SMs (at
    // least 16 blocks per CTA) rather than filling a few of them, since each
    // thread walks its blocks serially: 2,048 blocks run on 128 SMs, not 2
    const int64_t cap = device_sm_count();
    const int64_t want = std::max((P.total + dec_threads<G>() - 1) / dec_threads<G>(), (P.total + 15) / 16);
    const int grid = (int)(want < cap ? want : cap);
    decode_kernel<WIDE, MAXSEG, G><<<grid, dec_threads<G>(), dec_smem<G>(), s>>>(P);
    return cudaGetLastError();
}



bool wide_ok(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

}  // namespace

cudaError_t launch_decode(const ecco_tables* t, const uint8_t* blocks, const ecco_desc& d,
                          uint16_t* y, cudaStream_t s)
{
    DecParams<1> P;
    P.n_seg = 1;
    P.total = d.rows * d.groups_per_row;
    P.seg[0] = DecSeg{t->d, blocks, y, d, 0, P.total};
    return (wide_ok(y) && wide_ok(blocks)) ? run_decode<true, 1>(P, s) : run_decode<false, 1>(P, s);
}

cudaError_t launch_decode_act(const ecco_tables* t, const uint8_t* blocks, const ecco_desc& d,
                              uint16_t* y, cudaStream_t s)
{
    DecParams<1> P;
    P.n_seg = 1;
    P.total = d.rows * d.groups_per_row;
    P.seg[0] = DecSeg{t->d, blocks, y, d, 0, P.total};
    return (wide_ok(y) && wide_ok(blocks)) ? run_decode<true, 1, kGAct>(P, s) : run_decode<false, 1, kGAct>(P, s);
}

// Segments are packed into launches of at most kMultiSeg; empty ones are skipped.
cudaError_t launch_decode_multi(const ecco_segment* segs, int n, cudaStream_t s)
{
    constexpr int kMultiSeg = 64;
    int i = 0;
    while (i < n) {
        DecParams<kMultiSeg> P;
        P.n_seg = 0;
        P.total = 0;
        bool wide = true;
        while (i < n && P.n_seg < kMultiSeg) {
            const ecco_desc& d = segs[i].desc;
            const int64_t cnt = d.rows * d.groups_per_row;
            if (cnt > 0) {
                P.seg[P.n_seg++] = DecSeg{segs[i].tables->d, static_cast<const uint8_t*>(segs[i].src),
                                          static_cast<uint16_t*>(segs[i].dst), d, P.total, cnt};
                P.total += cnt;
                wide = wide && wide_ok(segs[i].dst) && wide_ok(segs[i].src);
            }
            ++i;
        }
        if (P.n_seg == 0) break;
        cudaError_t e = wide ? run_decode<true, kMultiSeg>(P, s) : run_decode<false, kMultiSeg>(P, s);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace ecco

// Device-side walker over one 512-bit block, shared by the decode and the
// fused decode+GEMV kernels.
//
// A thread owns one block.  The stream is consumed 8 symbols ("a chunk") at a
// time: two windows of 32 bits, each good for 4 codewords of at most 8 bits
// (the 8-bit limit of referee comment 1, Sec. 4.2 of the review page).  Each
// codeword costs one lookup in the codebook's 256-entry table (next 8 stream
// bits -> symbol | length << 4).  The chunk's 8 symbols come back as nibbles
// of one 32-bit word; their bf16 values are then selected from registers with
// byte permutes, 4 symbols per instruction, so the serial chain holds a single
// shared-memory load per symbol.
//
// Clipping: a chunk that starts with at least 64 bits of room cannot reach
// bit 512, so only chunks with less room count how many of their codewords
// end at or before bit 512; symbols from the first one that does not are
// reported as invalid (decoded as +0).
#pragma once

#include "ecco_internal.cuh"

namespace ecco {

// The 16 values bf16(s * C[p][j]) of one block as byte planes:
// lo[q] byte k = low byte of value 4q+k, hi[q] byte k = its high byte.
struct ValuePlanes {
    uint32_t lo[4], hi[4];
};

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);  // a -> low half, b -> high half
    return *reinterpret_cast<uint32_t*>(&v);
}

// Ct: centroids transposed, Ct[j * 64 + p], row 15 = 1.0 (the scale element);
// in shared memory, or read through the read-only cache when GLOBAL.
template <bool GLOBAL = false>
__device__ __forceinline__ ValuePlanes make_planes(float s, const float* Ct, int p)
{
    ValuePlanes v;
    auto c = [&](int j) { return GLOBAL ? __ldg(Ct + j * kNPat + p) : Ct[j * kNPat + p]; };
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint32_t a = pack_bf16x2(__fmul_rn(s, c(4 * q + 0)), __fmul_rn(s, c(4 * q + 1)));
        uint32_t b = pack_bf16x2(__fmul_rn(s, c(4 * q + 2)), __fmul_rn(s, c(4 * q + 3)));
        v.lo[q] = __byte_perm(a, b, 0x6420);
        v.hi[q] = __byte_perm(a, b, 0x7531);
    }
    return v;
}

// PTX prmt in its default mode: a selector nibble with bit 3 set replicates
// the sign bit of the byte it picks across the output byte.
__device__ __forceinline__ uint32_t prmt_sign(uint32_t x, uint32_t y, uint32_t sel)
{
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(x), "r"(y), "r"(sel));
    return r;
}

// Values of 4 symbols held in nibbles 4h..4h+3 of `nib` -> two bf16x2 words.
template <int H>
__device__ __forceinline__ void planes_to_bf16(const ValuePlanes& v, uint32_t nib, uint32_t nib_sh4,
                                               uint32_t& w0, uint32_t& w1)
{
    const uint32_t sel = (H == 0 ? nib : (nib >> 16)) & 0x7777u;  // byte index inside a half table
    // 0xff in byte k where symbol k >= 8 (bit 3 of its nibble): sign-replicating permute
    const uint32_t m = prmt_sign(nib_sh4, nib, H == 0 ? 0xD9C8u : 0xFBEAu);
    uint32_t lo = (__byte_perm(v.lo[0], v.lo[1], sel) & ~m) | (__byte_perm(v.lo[2], v.lo[3], sel) & m);
    uint32_t hi = (__byte_perm(v.hi[0], v.hi[1], sel) & ~m) | (__byte_perm(v.hi[2], v.hi[3], sel) & m);
    w0 = __byte_perm(lo, hi, 0x5140);
    w1 = __byte_perm(lo, hi, 0x7362);
}

// Stream position of one block.  Words 0..1 live in registers, words 2..15 in
// shared memory at ws[k * stride] (the thread's own column: conflict-free).
struct Stream {
    uint32_t lo, hi;  // 64-bit window, bit b of (hi:lo) is the next stream bit
    int b;            // 0 <= b < 32 at chunk boundaries
    int widx;         // next word to bring into the window
    int room;         // bits left before bit 512 (negative once clipped)
};

__device__ __forceinline__ void refill(Stream& st, const uint32_t* ws, int stride)
{
    if (st.b >= 32) {
        st.lo = st.hi;
        st.hi = (st.widx < 16) ? ws[st.widx * stride] : 0u;
        st.widx++;
        st.b -= 32;
    }
}

// Shared-memory key of a block's decode table: the table's address (tables
// start on a 256-byte boundary of the shared window, see aligned_smem) OR-ed
// with its swizzle.  `hdr` = header bits 8..15 = codebook * 64 + pattern, the
// table index.  Entry e of table t sits at byte e ^ ((t & 31) << 2): its
// 4-byte word is XOR-ed with the low 5 bits of t, so lanes that read the same
// entry of different tables -- common, since canonical codes give the short,
// frequent codewords the same low stream bits in every codebook -- land in
// different banks.  (ecco_tables.cu builds the tables in this layout.)
__device__ __forceinline__ uint32_t lut_key(const uint8_t* s_lut, uint32_t hdr)
{
    return ((uint32_t)__cvta_generic_to_shared(s_lut) + hdr * 256u) | ((hdr & 31u) << 2);
}

// Decodes 8 symbols.  Returns their nibbles (symbol k in bits 4k..4k+3); `kv`
// = number of them that end
// at or before bit 512 (8 unless CHECK and the block clips here or earlier).
// `lkey` = lut_key() of the block's table: the lookup address is the key
// XOR-ed with the next 8 stream bits.
template <bool CHECK>
__device__ __forceinline__ uint32_t decode8(Stream& st, uint32_t lkey, const uint32_t* ws, int stride, int& kv)
{
    uint32_t nib = 0;
    int used = 0;
    kv = 0;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        refill(st, ws, stride);
        uint32_t cur = __funnelshift_r(st.lo, st.hi, st.b);
        int u = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            // volatile with a memory clobber: the load stays on its side of
            // the barriers around the tables' staging
            uint32_t e;
            asm volatile("ld.shared.u8 %0, [%1];" : "=r"(e) : "r"(lkey ^ (cur & 0xffu)) : "memory");
            uint32_t len = e >> 4;
            nib = __funnelshift_r(nib, e, 4);  // symbol into the top nibble; the first ends at the bottom
            cur >>= len;
            u += (int)len;
            if (CHECK) kv += (used + u <= st.room) ? 1 : 0;
        }
        st.b += u;
        used += u;
    }
    if (!CHECK) kv = 8;
    st.room -= used;
    return nib;
}

// Keeps the first kv (0..8) bf16 values of a chunk's 4 output words.
__device__ __forceinline__ void mask_tail(uint32_t w[4], int kv)
{
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        int bits = min(max(16 * kv - 32 * q, 0), 32);
        uint32_t keep = (bits >= 32) ? 0xffffffffu : ((1u << bits) - 1u);
        w[q] &= keep;
    }
}

// Decodes one chunk into 4 bf16x2 words; also returns the nibbles.  The
// lanes that run together take the checked walk as soon as one of them is
// within 64 bits of the end (a vote), so a warp never runs both walks.
__device__ __forceinline__ uint32_t chunk_values(Stream& st, uint32_t lkey, const uint32_t* ws, int stride,
                                                 const ValuePlanes& vp, uint32_t w[4])
{
    int kv;
    uint32_t nib;
    if (__any_sync(__activemask(), st.room < 64))
        nib = decode8<true>(st, lkey, ws, stride, kv);
    else
        nib = decode8<false>(st, lkey, ws, stride, kv);
    uint32_t sh4 = nib << 4;
    planes_to_bf16<0>(vp, nib, sh4, w[0], w[1]);
    planes_to_bf16<1>(vp, nib, sh4, w[2], w[3]);
    if (kv < 8) mask_tail(w, kv);
    return nib;
}

// q / 127 correctly rounded (the outlier record's value, R15), without a
// division: x0 = q * r with r = RN(1/127), the residual q - 127 x0 is exact
// in one fused multiply-add, and one more gives the rounded quotient
// (Markstein's correction step for division by a constant; checked against
// the exactly rounded quotient for all 255 values of q, and bit-exact against
// the oracle's IEEE division in the parity tests).
__device__ __forceinline__ float q_over_127(int q)
{
    const float r = __uint_as_float(0x3c010204u);  // RN(1 / 127)
    const float qf = (float)q;
    const float x0 = __fmul_rn(qf, r);
    const float res = __fmaf_rn(-x0, 127.0f, qf);
    return __fmaf_rn(res, r, x0);
}

// Reads the 15-bit outlier record starting at stream bit `at` (>= 64).
__device__ __forceinline__ uint32_t read_record(const uint32_t* ws, int stride, int at)
{
    int wi = at >> 5;
    uint32_t w0 = ws[wi * stride];
    uint32_t w1 = (wi + 1 < 16) ? ws[(wi + 1) * stride] : 0u;
    return __funnelshift_r(w0, w1, at & 31) & 0x7fffu;
}

__device__ __forceinline__ void stage_words(uint32_t* ws, int stride, const uint4& q0, const uint4& q1,
                                            const uint4& q2, const uint4& q3)
{
    ws[2 * stride] = q0.z;
    ws[3 * stride] = q0.w;
    ws[4 * stride] = q1.x;
    ws[5 * stride] = q1.y;
    ws[6 * stride] = q1.z;
    ws[7 * stride] = q1.w;
    ws[8 * stride] = q2.x;
    ws[9 * stride] = q2.y;
    ws[10 * stride] = q2.z;
    ws[11 * stride] = q2.w;
    ws[12 * stride] = q3.x;
    ws[13 * stride] = q3.y;
    ws[14 * stride] = q3.z;
    ws[15 * stride] = q3.w;
}

// Kernels that walk blocks reserve kSmemAlign bytes more than their layout
// needs and lay it out from aligned_smem(): the decode tables then start on a
// 256-byte boundary of the shared window, as decode8 requires.
constexpr size_t kSmemAlign = 256;

__device__ __forceinline__ uint8_t* aligned_smem(uint8_t* raw)
{
    const uint32_t a = (uint32_t)__cvta_generic_to_shared(raw);
    return raw + ((uint32_t)kSmemAlign - (a & ((uint32_t)kSmemAlign - 1u))) % (uint32_t)kSmemAlign;
}

// Copies a tensor's decode tables (65,536 B) and transposed centroids (4,096 B)
// into shared memory with every 16-byte load issued before any store.
template <int NT>
__device__ __forceinline__ void stage_tables(const DevTables* tb, uint8_t* s_lut, float* s_Ct, int tid)
{
    constexpr int kLutVec = (int)(sizeof(((DevTables*)0)->lut) / 16);
    constexpr int kCtVec = (int)(sizeof(((DevTables*)0)->Ct) / 16);
    constexpr int kAll = kLutVec + kCtVec;
    constexpr int kPer = (kAll + NT - 1) / NT;
    const uint4* lut = reinterpret_cast<const uint4*>(&tb->lut[0][0]);
    const uint4* ct = reinterpret_cast<const uint4*>(&tb->Ct[0][0]);
    uint4 v[kPer];
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
        const int i = tid + k * NT;
        if (i < kAll) v[k] = __ldg(i < kLutVec ? lut + i : ct + (i - kLutVec));
    }
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
        const int i = tid + k * NT;
        if (i < kLutVec)
            reinterpret_cast<uint4*>(s_lut)[i] = v[k];
        else if (i < kAll)
            reinterpret_cast<uint4*>(s_Ct)[i - kLutVec] = v[k];
    }
}

// Copies a tensor's decode tables alone (65,536 B), every 16-byte load issued
// before any store (kernels that read the centroids through the read-only
// cache instead).
template <int NT>
__device__ __forceinline__ void stage_lut(const DevTables* tb, uint8_t* s_lut, int tid)
{
    constexpr int kLutVec = (int)(sizeof(((DevTables*)0)->lut) / 16);
    constexpr int kPer = (kLutVec + NT - 1) / NT;
    const uint4* lut = reinterpret_cast<const uint4*>(&tb->lut[0][0]);
    uint4 v[kPer];
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
        const int i = tid + k * NT;
        if (i < kLutVec) v[k] = __ldg(lut + i);
    }
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
        const int i = tid + k * NT;
        if (i < kLutVec) reinterpret_cast<uint4*>(s_lut)[i] = v[k];
    }
}

__device__ __forceinline__ void stg256(void* p, const uint32_t a[4], const uint32_t b[4])
{
    asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(a[0]), "r"(a[1]),
                 "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]), "r"(b[2]), "r"(b[3])
                 : "memory");
}

}  // namespace ecco

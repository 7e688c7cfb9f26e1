// da2_prepare.cu -- fused operand preparation ("DraftAttention2", Sec. 3.3
// "Fused quantization and reordering", Fig. 3b; Eq. 2; App. C.1 formats).
//
// One CTA per (64-token block a, head, tensor).  It gathers the block's
// tokens through the partition (one coalesced 16-byte load per 8 channels of
// a token row; all of a thread's loads are issued before the first is used),
// then from the staged tile writes in a single pass:
//   Q/K: pooled descriptors (fp64 mean over the valid slots, summed in slot
//        order, and channel max; Eq. 2), FP8 e4m3 codes with the tile scale
//        amax/448, two-level NVFP4 codes (tile scale amax/2688, ue4m3 scale
//        per 16 channels);
//   V:   the transposed tile (V^T, value transposition folded into packing)
//        quantized the same way with NVFP4 groups of 16 slots, and the
//        per-head maxima of the V tile scales.
// Optional extra outputs: the bf16 tiles of the 16-bit path (Q, K and V^T as
// they are) and the INT8 tiles of the 8-bit phase's QK^T (Q and K; scale
// amax/127, codes RNE(x * (127/amax)) clamped to +-127).
// Operand tiles are written directly in the tcgen05 K-major no-swizzle
// layout (core matrices of 8 rows x 16 bytes), so the attention kernel moves
// each tile with one bulk copy.  Every quantizer step is an fp32
// round-to-nearest operation followed by the hardware RNE-satfinite
// converter.
#include "da2_common.cuh"
#include "da2_kernels.h"

namespace da2 {

namespace {

// threads per CTA: one quantization item (32 elements of an operand row) per thread
template <int D>
constexpr int threads_for() { return D == 64 ? 128 : 256; }
// Resident CTAs per SM the register budget must allow: enough 16 KB tiles in
// flight per SM to cover the memory latency (4 x 256 or 8 x 128 threads,
// 64 registers each).
template <int D>
constexpr int min_ctas_for() { return D == 64 ? 8 : 4; }

// Byte offset of 16-byte chunk `chunk` of row `row` in a K-major
// no-swizzle operand tile with `row_bytes` bytes per row: core matrices of
// 8 rows x 16 bytes, adjacent along K, then along the rows.
__device__ __forceinline__ uint32_t kmajor_offset(int row, int chunk, int row_bytes) {
    return ((row >> 3) * (row_bytes >> 4) + chunk) * 128 + (row & 7) * 16;
}

// Largest |x| of the bf16 pairs in n words, per half: |x| of a finite bf16
// orders like its 15 magnitude bits.
template <int N>
__device__ __forceinline__ uint32_t absmax_bf16x2(const uint32_t* w) {
    uint32_t m = w[0] & 0x7FFF7FFFu;
#pragma unroll
    for (int i = 1; i + 1 < N; i += 2) m = __vimax3_u16x2(m, w[i] & 0x7FFF7FFFu, w[i + 1] & 0x7FFF7FFFu);
    if constexpr (N % 2 == 0) m = __vmaxu2(m, w[N - 1] & 0x7FFF7FFFu);
    return m;
}

template <int D>
__global__ void __launch_bounds__(threads_for<D>(), min_ctas_for<D>()) prepare_kernel(PrepareArgs p) {
    constexpr int kThreads = threads_for<D>();
    constexpr int LD = D + 8;  // padded smem row (bf16 elements) against bank conflicts
    __shared__ __align__(16) uint16_t tile[64 * LD];
    __shared__ int tok[64];
    __shared__ float warp_max[kThreads / 32];
    __shared__ __align__(16) uint8_t sf_atom[512];

    const int a = blockIdx.x, bh = blockIdx.y, which = blockIdx.z;  // which: 0 Q, 1 K, 2 V
    const int tid = threadIdx.x;
    const int R = p.R, BH = p.B * p.H;
    const int b = bh / p.H, h = bh % p.H;
    const size_t ba = (size_t)bh * R + a;

    if (tid < 64) tok[tid] = p.slot_token[a * 64 + tid];
    for (int i = tid; i < 128; i += kThreads) reinterpret_cast<uint32_t*>(sf_atom)[i] = 0u;
    __syncthreads();

    // ---- gather: 64 rows x D/8 chunks of 16 bytes
    const __nv_bfloat16* src = which == 0 ? p.q : (which == 1 ? p.k : p.v);
    src += (size_t)b * p.s0 + (size_t)h * p.s1;
    float amax = 0.0f;
    constexpr int kChunks = 64 * (D / 8) / kThreads;  // 16-byte loads per thread
    static_assert(kChunks * kThreads == 64 * (D / 8), "whole chunks per thread");
    uint4 val[kChunks];
#pragma unroll
    for (int u = 0; u < kChunks; ++u) {
        const int i = tid + u * kThreads, r = i / (D / 8), c8 = i % (D / 8);
        const int t = tok[r];
        val[u] = t >= 0 ? __ldg(reinterpret_cast<const uint4*>(src + (size_t)t * p.s2 + c8 * 8))
                        : make_uint4(0, 0, 0, 0);
    }
    // |x| of a finite bf16 orders like its 15 magnitude bits, so the tile
    // maximum is taken on the bits, two halves per instruction
    uint32_t mag2 = 0u;
#pragma unroll
    for (int u = 0; u < kChunks; ++u) {
        const int i = tid + u * kThreads, r = i / (D / 8), c8 = i % (D / 8);
        *reinterpret_cast<uint4*>(&tile[r * LD + c8 * 8]) = val[u];
        mag2 = __vmaxu2(mag2, __vmaxu2(val[u].x & 0x7FFF7FFFu, val[u].y & 0x7FFF7FFFu));
        mag2 = __vmaxu2(mag2, __vmaxu2(val[u].z & 0x7FFF7FFFu, val[u].w & 0x7FFF7FFFu));
    }
    amax = __uint_as_float(max(mag2 & 0xFFFFu, mag2 >> 16) << 16);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if ((tid & 31) == 0) warp_max[tid >> 5] = amax;
    __syncthreads();
    amax = warp_max[0];
#pragma unroll
    for (int w = 1; w < kThreads / 32; ++w) amax = fmaxf(amax, warp_max[w]);

    auto X = [&](int r, int c) -> float { return bf16_bits_to_f32(tile[r * LD + c]); };

    // ---- pooled descriptors (Eq. 2), Q and K only: thread c < D sums column c
    // in fp64 in slot order, thread D + c takes its maximum (exact in fp32, the
    // values are bf16), so each thread runs one dependency chain
    static_assert(kThreads >= 2 * D, "a sum thread and a max thread per channel");
    if (which < 2 && tid < 2 * D) {
        const int na = p.n_a[a];
        const int c = tid < D ? tid : tid - D;
        const size_t plane = (size_t)BH * R * D;
        if (tid < D) {
            double s = 0.0;
#pragma unroll 8
            for (int j = 0; j < na; ++j) s += (double)X(j, c);
            p.desc[(2 * which) * plane + ba * D + c] = s / (double)na;
        } else {
            float m = X(0, c);
#pragma unroll 8
            for (int j = 1; j < na; ++j) m = fmaxf(m, X(j, c));
            p.desc[(2 * which + 1) * plane + ba * D + c] = (double)m;
        }
    }

    // ---- scales
    const bool zero = (amax == 0.0f);
    const float s8 = zero ? 0.0f : __fdiv_rn(amax, 448.0f);
    const float inv8 = zero ? 0.0f : __fdiv_rn(448.0f, amax);
    const float g4 = zero ? 0.0f : __fdiv_rn(amax, 2688.0f);
    const float t4 = zero ? 0.0f : __fdiv_rn(448.0f, amax);
    const float inv8i = zero ? 0.0f : __fdiv_rn(127.0f, amax);
    if (tid == 0) {
        p.scale[(size_t)which * BH * R + ba] = s8;
        p.scale[(size_t)(3 + which) * BH * R + ba] = g4;
        if (p.si8 && which < 2) p.si8[(size_t)which * BH * R + ba] = zero ? 0.0f : __fdiv_rn(amax, 127.0f);
        if (which == 2 && a < p.Rv) {  // the phase units cover the video blocks
            atomicMax(reinterpret_cast<unsigned*>(&p.vmax[bh]), __float_as_uint(s8));
            atomicMax(reinterpret_cast<unsigned*>(&p.vmax[BH + bh]), __float_as_uint(g4));
        }
    }

    // Quantized operand matrices, written in the K-major core-matrix layout:
    // Q/K rows are the 64 slots (cols = D channels), V^T rows are the D
    // channels (cols = 64 slots).  Each work item quantizes 32 consecutive
    // elements of one row to FP8 (two 16-byte chunks) and NVFP4 (one 16-byte
    // chunk, two scale bytes) from registers.
    uint8_t* dst8 = (which == 0 ? p.q8 : (which == 1 ? p.k8 : p.v8)) + ba * (size_t)(64 * D);
    uint8_t* dst4 = (which == 0 ? p.q4 : (which == 1 ? p.k4 : p.v4)) + ba * (size_t)(32 * D);
    // FP8 e4m3 of 16 values: e4m3(RN(x * inv8)), 0 for a zero tile
    auto fp8x16 = [&](const float* x) -> uint4 {
        if (zero) return make_uint4(0u, 0u, 0u, 0u);
        const float2 s2 = make_float2(inv8, inv8);
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
            w[e] = pack_e4m3x4(__fmul2_rn(make_float2(x[4 * e], x[4 * e + 1]), s2),
                               __fmul2_rn(make_float2(x[4 * e + 2], x[4 * e + 3]), s2));
        return make_uint4(w[0], w[1], w[2], w[3]);
    };
    // NVFP4 group of 16 values with largest magnitude a16: scale byte
    // sf = e4m3(RN(a16 * 448/amax)), codes e2m1(RN(x * RN(1 / RN(value(sf) * g4))))
    // into 8 bytes
    auto fp4x16 = [&](const float* x, float a16, uint8_t* sf_out) -> uint2 {
        const uint32_t sf = zero ? 0u : (uint32_t)(cvt_e4m3x2(__fmul_rn(a16, t4), 0.0f) & 0xFF);
        *sf_out = (uint8_t)sf;
        if (sf == 0) return make_uint2(0u, 0u);
        const float rcp = __frcp_rn(__fmul_rn(e4m3_to_f32((uint8_t)sf), g4));
        const float2 r2 = make_float2(rcp, rcp);
        auto y = [&](int i) { return __fmul2_rn(make_float2(x[i], x[i + 1]), r2); };
        return make_uint2(pack_e2m1x8(y(0), y(2), y(4), y(6)), pack_e2m1x8(y(8), y(10), y(12), y(14)));
    };
    auto bf_lo = [](uint32_t w) { return __uint_as_float(w << 16); };
    auto bf_hi = [](uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); };

    if (which < 2) {
        // item (slot r, 32-channel chunk k); a warp covers 32 consecutive slots
        // of one chunk: its 16-byte shared reads fall in distinct banks
        for (int it = tid; it < 64 * (D / 32); it += kThreads) {
            const int r = it & 63, k = it >> 6;
            float x[32];
            uint32_t ww[16];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint4 raw = *reinterpret_cast<const uint4*>(&tile[r * LD + 32 * k + 8 * q]);
                ww[4 * q] = raw.x;
                ww[4 * q + 1] = raw.y;
                ww[4 * q + 2] = raw.z;
                ww[4 * q + 3] = raw.w;
            }
            // largest magnitude of each 16-channel group (8 words each)
            const uint32_t m0 = absmax_bf16x2<8>(ww), m1 = absmax_bf16x2<8>(ww + 8);
            const float a0 = __uint_as_float(max(m0 & 0xFFFFu, m0 >> 16) << 16);
            const float a1 = __uint_as_float(max(m1 & 0xFFFFu, m1 >> 16) << 16);
            if (p.q16) {
                // bf16 tile of the 16-bit path: the input values as they are (2D-byte rows)
                uint8_t* dst16 = (which == 0 ? p.q16 : p.k16) + ba * (size_t)(128 * D);
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    *reinterpret_cast<uint4*>(dst16 + kmajor_offset(r, 4 * k + q, 2 * D)) =
                        make_uint4(ww[4 * q], ww[4 * q + 1], ww[4 * q + 2], ww[4 * q + 3]);
            }
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                x[2 * e] = bf_lo(ww[e]);
                x[2 * e + 1] = bf_hi(ww[e]);
            }
            if (p.q8i) {
                int8_t* dsti = (which == 0 ? p.q8i : p.k8i) + ba * (size_t)(64 * D);
                uint32_t wi[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    uint32_t acc = 0;
#pragma unroll
                    for (int b4 = 0; b4 < 4; ++b4) {
                        int c = zero ? 0 : __float2int_rn(__fmul_rn(x[4 * e + b4], inv8i));
                        c = c > 127 ? 127 : (c < -127 ? -127 : c);
                        acc |= ((uint32_t)c & 0xFFu) << (8 * b4);
                    }
                    wi[e] = acc;
                }
                *reinterpret_cast<uint4*>(dsti + kmajor_offset(r, 2 * k, D)) = make_uint4(wi[0], wi[1], wi[2], wi[3]);
                *reinterpret_cast<uint4*>(dsti + kmajor_offset(r, 2 * k + 1, D)) = make_uint4(wi[4], wi[5], wi[6], wi[7]);
            }
            *reinterpret_cast<uint4*>(dst8 + kmajor_offset(r, 2 * k, D)) = fp8x16(x);
            *reinterpret_cast<uint4*>(dst8 + kmajor_offset(r, 2 * k + 1, D)) = fp8x16(x + 16);
            uint8_t sf0, sf1;
            const uint2 c0 = fp4x16(x, a0, &sf0), c1 = fp4x16(x + 16, a1, &sf1);
            *reinterpret_cast<uint4*>(dst4 + kmajor_offset(r, k, D / 2)) = make_uint4(c0.x, c0.y, c1.x, c1.y);
#pragma unroll
            for (int gi = 0; gi < 2; ++gi) {
                const int gcol = 2 * k + gi;  // group index along the row
                const uint8_t sf = gi ? sf1 : sf0;
                if (which == 0) sf_atom[r * (D / 16) + gcol] = sf;
                else sf_atom[16 * (r & 31) + 4 * (2 * (gcol / 4) + (r >> 5)) + (gcol % 4)] = sf;
            }
        }
    } else {
        // V^T: item (channel pair 2c, 2c+1; 16-slot group k); one 32-bit shared
        // read gives both channels of a slot, a warp reads 128 contiguous bytes
        for (int it = tid; it < (D / 2) * 4; it += kThreads) {
            const int c = it % (D / 2), k = it / (D / 2);
            uint32_t w[16];  // slot sl of the group: channel 2c in the low half, 2c+1 in the high half
#pragma unroll
            for (int sl = 0; sl < 16; ++sl) w[sl] = *reinterpret_cast<const uint32_t*>(&tile[(16 * k + sl) * LD + 2 * c]);
            if (p.v16) {
                // bf16 V^T of the 16-bit path: rows 2c and 2c+1, 32 bytes each (128-byte rows)
                uint8_t* dst16 = p.v16 + ba * (size_t)(128 * D);
                uint32_t b16[2][8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    b16[0][i] = __byte_perm(w[2 * i], w[2 * i + 1], 0x5410);
                    b16[1][i] = __byte_perm(w[2 * i], w[2 * i + 1], 0x7632);
                }
#pragma unroll
                for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                    for (int q = 0; q < 2; ++q)
                        *reinterpret_cast<uint4*>(dst16 + kmajor_offset(2 * c + hh, 2 * k + q, 128)) =
                            make_uint4(b16[hh][4 * q], b16[hh][4 * q + 1], b16[hh][4 * q + 2], b16[hh][4 * q + 3]);
            }
            // largest magnitude of the group in each channel
            const uint32_t m2 = absmax_bf16x2<16>(w);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int row = 2 * c + h;
                float x[16];
#pragma unroll
                for (int sl = 0; sl < 16; ++sl) x[sl] = h ? bf_hi(w[sl]) : bf_lo(w[sl]);
                *reinterpret_cast<uint4*>(dst8 + kmajor_offset(row, k, 64)) = fp8x16(x);
                uint8_t sf;
                const float a16 = __uint_as_float((h ? m2 >> 16 : m2 & 0xFFFFu) << 16);
                const uint2 c4 = fp4x16(x, a16, &sf);
                *reinterpret_cast<uint2*>(dst4 + kmajor_offset(row, k >> 1, 32) + 8 * (k & 1)) = c4;
                sf_atom[16 * (row & 31) + 4 * (row >> 5) + k] = sf;
            }
        }
    }
    __syncthreads();
    // ---- scale factors: Q row-major [64][D/16]; K, V one 512-byte atom
    {
        uint8_t* dst;
        int bytes;
        if (which == 0) {
            dst = p.sfq + ba * (size_t)(64 * (D / 16));
            bytes = 64 * (D / 16);
        } else {
            dst = (which == 1 ? p.sfk : p.sfv) + ba * (size_t)512;
            bytes = 512;
        }
        for (int i = tid; i < bytes / 16; i += kThreads)
            reinterpret_cast<uint4*>(dst)[i] = reinterpret_cast<const uint4*>(sf_atom)[i];
    }
}

}  // namespace

cudaError_t launch_prepare(const PrepareArgs& p, cudaStream_t stream) {
    const int BH = p.B * p.H;
    cudaError_t e = cudaMemsetAsync(p.vmax, 0, sizeof(float) * 2 * BH, stream);
    if (e != cudaSuccess) return e;
    dim3 grid(p.R, BH, 3);
    if (p.d == 64) prepare_kernel<64><<<grid, threads_for<64>(), 0, stream>>>(p);
    else prepare_kernel<128><<<grid, threads_for<128>(), 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace da2

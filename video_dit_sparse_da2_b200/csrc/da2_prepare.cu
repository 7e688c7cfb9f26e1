// da2_prepare.cu -- fused operand preparation ("DraftAttention2", Sec. 3.3
// "Fused quantization and reordering", Fig. 3b; Eq. 2; App. C.1 formats).
//
// One CTA per (64-token block a, head, tensor).  It gathers the block's
// tokens through the partition (one coalesced 16-byte load per 8 channels of
// a token row), then from the staged tile writes in a single pass:
//   Q/K: pooled descriptors (fp64 mean over the valid slots, summed in slot
//        order, and channel max; Eq. 2), FP8 e4m3 codes with the tile scale
//        amax/448, two-level NVFP4 codes (tile scale amax/2688, ue4m3 scale
//        per 16 channels);
//   V:   the transposed tile (V^T, value transposition folded into packing)
//        quantized the same way with NVFP4 groups of 16 slots, and the
//        per-head maxima of the V tile scales.
// Operand tiles are written directly in the tcgen05 K-major no-swizzle
// layout (core matrices of 8 rows x 16 bytes), so the attention kernel moves
// each tile with one bulk copy.  Every quantizer step is an fp32
// round-to-nearest operation followed by the hardware RNE-satfinite
// converter.
#include "da2_common.cuh"
#include "da2_kernels.h"

namespace da2 {

namespace {

constexpr int kThreads = 256;

template <int D>
__global__ void __launch_bounds__(kThreads) prepare_kernel(PrepareArgs p) {
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
    for (int i = tid; i < 64 * (D / 8); i += kThreads) {
        const int r = i / (D / 8), c8 = i % (D / 8);
        const int t = tok[r];
        uint4 val = make_uint4(0, 0, 0, 0);
        if (t >= 0) val = __ldg(reinterpret_cast<const uint4*>(src + (size_t)t * p.s2 + c8 * 8));
        *reinterpret_cast<uint4*>(&tile[r * LD + c8 * 8]) = val;
        const uint32_t w[4] = {val.x, val.y, val.z, val.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            amax = fmaxf(amax, fabsf(__uint_as_float(w[e] << 16)));
            amax = fmaxf(amax, fabsf(__uint_as_float(w[e] & 0xFFFF0000u)));
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if ((tid & 31) == 0) warp_max[tid >> 5] = amax;
    __syncthreads();
    amax = warp_max[0];
#pragma unroll
    for (int w = 1; w < kThreads / 32; ++w) amax = fmaxf(amax, warp_max[w]);

    auto X = [&](int r, int c) -> float { return bf16_bits_to_f32(tile[r * LD + c]); };

    // ---- pooled descriptors (Eq. 2), Q and K only
    if (which < 2 && tid < D) {
        const int na = p.n_a[a];
        double s = 0.0, m = (double)X(0, tid);
        for (int j = 0; j < na; ++j) {
            const double x = (double)X(j, tid);
            s += x;
            m = fmax(m, x);
        }
        const size_t plane = (size_t)BH * R * D;
        p.desc[(2 * which) * plane + ba * D + tid] = s / (double)na;
        p.desc[(2 * which + 1) * plane + ba * D + tid] = m;
    }

    // ---- scales
    const bool zero = (amax == 0.0f);
    const float s8 = zero ? 0.0f : __fdiv_rn(amax, 448.0f);
    const float inv8 = zero ? 0.0f : __fdiv_rn(448.0f, amax);
    const float g4 = zero ? 0.0f : __fdiv_rn(amax, 2688.0f);
    const float t4 = zero ? 0.0f : __fdiv_rn(448.0f, amax);
    if (tid == 0) {
        p.scale[(size_t)which * BH * R + ba] = s8;
        p.scale[(size_t)(3 + which) * BH * R + ba] = g4;
        if (which == 2) {
            atomicMax(reinterpret_cast<unsigned*>(&p.vmax[bh]), __float_as_uint(s8));
            atomicMax(reinterpret_cast<unsigned*>(&p.vmax[BH + bh]), __float_as_uint(g4));
        }
    }

    // Element (row, col) of the operand matrix: Q/K are the tile itself
    // (rows = slots), V is transposed (rows = channels, cols = slots).
    const bool vt = (which == 2);
    const int rows = vt ? D : 64;
    const int cols = vt ? 64 : D;
    auto E = [&](int r, int c) -> float { return vt ? X(c, r) : X(r, c); };

    // ---- FP8: cols bytes per row, chunks of 16 in memory order
    {
        uint8_t* dst = (which == 0 ? p.q8 : (which == 1 ? p.k8 : p.v8)) + ba * (size_t)(64 * D);
        const int cpr = cols / 16;
        for (int m = tid; m < rows * cpr; m += kThreads) {
            const int grp = m / (8 * cpr), rem = m % (8 * cpr);
            const int chunk = rem / 8, r = grp * 8 + (rem % 8);
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int c = chunk * 16 + e * 4;
                const uint16_t lo = zero ? 0 : cvt_e4m3x2(__fmul_rn(E(r, c), inv8), __fmul_rn(E(r, c + 1), inv8));
                const uint16_t hi =
                    zero ? 0 : cvt_e4m3x2(__fmul_rn(E(r, c + 2), inv8), __fmul_rn(E(r, c + 3), inv8));
                w[e] = (uint32_t)lo | ((uint32_t)hi << 16);
            }
            *reinterpret_cast<uint4*>(dst + (size_t)m * 16) = make_uint4(w[0], w[1], w[2], w[3]);
        }
    }

    // ---- NVFP4: cols/2 bytes per row; one 16-byte chunk = 32 elements = 2 groups
    {
        uint8_t* dst = (which == 0 ? p.q4 : (which == 1 ? p.k4 : p.v4)) + ba * (size_t)(32 * D);
        const int cpr = cols / 32;
        for (int m = tid; m < rows * cpr; m += kThreads) {
            const int grp = m / (8 * cpr), rem = m % (8 * cpr);
            const int chunk = rem / 8, r = grp * 8 + (rem % 8);
            uint8_t bytes[16];
#pragma unroll
            for (int gi = 0; gi < 2; ++gi) {
                const int c0 = chunk * 32 + gi * 16;
                float v[16], a16 = 0.0f;
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    v[e] = E(r, c0 + e);
                    a16 = fmaxf(a16, fabsf(v[e]));
                }
                uint8_t sf = 0;
                if (!zero) sf = (uint8_t)(cvt_e4m3x2(__fmul_rn(a16, t4), 0.0f) & 0xFF);
                const float rcp = sf ? __fdiv_rn(1.0f, __fmul_rn(e4m3_to_f32(sf), g4)) : 0.0f;
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    bytes[gi * 8 + e] = sf ? cvt_e2m1x2(__fmul_rn(v[2 * e], rcp), __fmul_rn(v[2 * e + 1], rcp)) : 0;
                // scale byte: group index along the row is c0/16
                const int gcol = c0 / 16;
                if (which == 0) {
                    sf_atom[r * (D / 16) + gcol] = sf;
                } else if (which == 1) {
                    sf_atom[16 * (r & 31) + 4 * (2 * (c0 / 64) + (r >> 5)) + (c0 % 64) / 16] = sf;
                } else {
                    sf_atom[16 * (r & 31) + 4 * (r >> 5) + gcol] = sf;
                }
            }
            uint4 out;
            memcpy(&out, bytes, 16);
            *reinterpret_cast<uint4*>(dst + (size_t)m * 16) = out;
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
    if (p.d == 64) prepare_kernel<64><<<grid, kThreads, 0, stream>>>(p);
    else prepare_kernel<128><<<grid, kThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace da2

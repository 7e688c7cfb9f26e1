// da2_plan_mx.cu -- the max-pool branch of the draft logits (DraftAttention2
// Eq. 3) from exact integer tensor-core products.
//
// The draft defines a logit as an fp64 fma chain over the channels in
// ascending order, times 1/sqrt(d).  The max-pool descriptors are channel
// maxima of bf16 inputs, so every one of them is a bf16 value: sign, 8-bit
// significand M (with its leading bit) and exponent E.  Within a block (one
// row of the descriptor matrix) whose nonzero values span at most kMaxSpan
// binades above the smallest exponent e0, every value is N * 2^(e0 - 7) with
// an integer |N| < 2^21.  The product of two rows is then
// T * 2^(e0_a + e0_b - 14) with T = sum_c N_ac N_bc, |T| < 2^49; every partial
// sum of the defining fp64 chain is such an integer multiple below 2^53 units,
// so the chain is exact and equals T * 2^(...) exactly.  T itself is computed
// exactly by 8-bit tensor-core MMAs (tcgen05.mma kind::i8, s32 accumulation)
// on the split N = 2^14 h + 2^7 m + l (h in [-128, 127], m, l in [0, 127]):
// five accumulators collect the products of equal weight 2^28, 2^21, 2^14,
// 2^7 and 1 (h h', h m' + m h', h l' + m m' + l h', m l' + l m', l l').  The
// logit is then (double)T * 2^(e0_a + e0_b - 14) (exact) * (1/sqrt d), one
// rounding: bit for bit the defining value.  The rows and columns of the few
// blocks outside that range (or holding a value that is not a bf16 value)
// are recomputed by the fp64 chain itself (mx_strips_kernel).
#include "da2_common.cuh"
#include "da2_kernels.h"

namespace da2 {

namespace {

constexpr int kMaxSpan = 13;     // binades above e0: |N| <= 255 * 2^13 < 2^21
constexpr int kParts = 3;        // int8 parts of N: h, m, l
constexpr int kMxTile = 128;     // rows per split tile (the MMA's M)
constexpr int kMxN = 32;         // key blocks per MMA tile (the MMA's N)
constexpr int kAcc = 5;          // accumulators: weights 2^28, 2^21, 2^14, 2^7, 1
constexpr uint32_t kMxCols = 256;  // tensor-memory columns (kAcc x 32 used)
constexpr int kMxThreads = 128;
// dynamic shared memory: the parts of A (128 rows) and of B (32 rows), then
// the epilogue's staging rows (4 warps x 32 x 33 doubles)
template <int D>
constexpr int stage_off() { return kParts * (kMxTile + kMxN) * D; }
constexpr int kStageBytes = 4 * 32 * 33 * 8;
constexpr int kMxSmem = 96 * 1024;  // > 1/3 of an SM's shared memory: at most two CTAs per SM
static_assert(kParts * (kMxTile + kMxN) * 128 + kStageBytes <= kMxSmem, "tiles and staging fit");

__device__ __forceinline__ uint32_t kmajor_off_b(int row, int byte, int row_bytes) {
    return ((row >> 3) * (row_bytes >> 4) + (byte >> 4)) * 128 + (row & 7) * 16 + (byte & 15);
}

// 16 consecutive 32-bit columns of this warp's lanes, load and wait in one
// asm statement.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}

// One warp per descriptor row (block r of head bh, tensor t: 0 = Q max, 1 = K
// max): lane l handles channels 4l .. 4l+3.  Writes the three int8 parts in
// the tcgen05 K-major no-swizzle layout (128-row tiles), e0 and the row flag.
template <int D>
__global__ void __launch_bounds__(256) mx_split_kernel(PlanArgs p) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = blockIdx.x * 8 + warp, t = blockIdx.y, bh = blockIdx.z;
    const int Rp = p.mx_rpad, R = p.R;
    if (r >= Rp) return;
    const size_t plane = (size_t)p.BH * p.Rt * D;
    const double* row = p.desc + (size_t)(2 * t + 1) * plane + ((size_t)bh * p.Rt + r) * D;
    constexpr int kLanes = D / 4;
    int e[4] = {0, 0, 0, 0}, m[4] = {0, 0, 0, 0};
    bool nz[4] = {false, false, false, false};
    bool exact = true;
    int emin = 1 << 20, emax = -(1 << 20);
    if (r < R && lane < kLanes) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const unsigned long long bits = (unsigned long long)__double_as_longlong(row[4 * lane + i]);
            const int ex = (int)((bits >> 52) & 0x7FF);
            const unsigned long long mant = bits & 0xFFFFFFFFFFFFFull;
            if (ex == 0 && mant == 0) continue;  // +-0
            // a finite normal fp64 whose significand has at most 8 bits
            // (every bf16 value, subnormals included, is one)
            if (ex == 0 || ex == 0x7FF || (mant & ((1ull << 45) - 1)) != 0) {
                exact = false;
                continue;
            }
            nz[i] = true;
            e[i] = ex - 1023;
            m[i] = (int)(128 + (mant >> 45)) * ((bits >> 63) ? -1 : 1);
            emin = min(emin, e[i]);
            emax = max(emax, e[i]);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        emin = min(emin, __shfl_xor_sync(0xffffffffu, emin, o));
        emax = max(emax, __shfl_xor_sync(0xffffffffu, emax, o));
    }
    const bool ok = __all_sync(0xffffffffu, exact) && (emax < emin || emax - emin <= kMaxSpan);
    const int e0 = emax < emin ? 0 : emin;  // an all-zero row: every N is 0
    uint32_t w[kParts] = {0u, 0u, 0u};
    if (ok) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int N = nz[i] ? m[i] * (1 << (e[i] - e0)) : 0;
            const int h = N >> 14;                // floor: N = 2^14 h + rest, rest in [0, 2^14)
            const int rest = N - (h << 14);
            w[0] |= ((uint32_t)h & 0xFFu) << (8 * i);
            w[1] |= (uint32_t)(rest >> 7) << (8 * i);
            w[2] |= (uint32_t)(rest & 127) << (8 * i);
        }
    }
    // tiles [2][BH][Rp/128][part][128 * D]
    const size_t tile = ((size_t)t * p.BH + bh) * (Rp / kMxTile) + r / kMxTile;
    int8_t* base = p.mx_tiles + tile * kParts * kMxTile * D;
    if (lane < kLanes) {
        const uint32_t o = kmajor_off_b(r % kMxTile, 4 * lane, D);
#pragma unroll
        for (int q = 0; q < kParts; ++q) *reinterpret_cast<uint32_t*>(base + q * kMxTile * D + o) = w[q];
    }
    if (lane == 0) {
        const size_t ri = ((size_t)t * p.BH + bh) * Rp + r;
        p.mx_e0[ri] = e0;
        p.mx_ok[ri] = ok ? 1 : 0;
        if (!ok && r < R) p.mx_fail[1 + atomicAdd(&p.mx_fail[0], 1)] = (int)ri;
    }
}

// One CTA per (head, 128 query blocks, 32 key blocks): T of every pair from
// nine int8 products, then the logit; pairs whose query or key block is
// outside the exact range are left to mx_strips_kernel.
template <int D>
__global__ void __launch_bounds__(kMxThreads) mx_logits_kernel(PlanArgs p, double rd) {
    extern __shared__ __align__(1024) uint8_t sm[];
    __shared__ uint64_t bar_ld, bar_mma;
    __shared__ uint32_t tmem_sh;
    __shared__ int abort_sh;
    __shared__ int e0b_sh[kMxN];
    __shared__ uint8_t okb_sh[kMxN];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bt = blockIdx.x, at = blockIdx.y, bh = blockIdx.z;
    const int Rp = p.mx_rpad, R = p.R, BH = p.BH;
    const int a0 = at * kMxTile, b0 = bt * kMxN;
    const size_t ntile = Rp / kMxTile;
    const int8_t* qt = p.mx_tiles + ((size_t)bh * ntile + at) * kParts * kMxTile * D;
    const int8_t* kt = p.mx_tiles + (((size_t)BH + bh) * ntile + b0 / kMxTile) * kParts * kMxTile * D;
    const size_t kslice = (size_t)(b0 % kMxTile) * D;  // rows b0 % 128 .. +31 of the K tile
    volatile int* abort_v = &abort_sh;
    if (threadIdx.x == 0) {
        mbar_init(&bar_ld, 1);
        mbar_init(&bar_mma, 1);
        abort_sh = 0;
        fence_mbar_init();
    }
    if (threadIdx.x < kMxN) {
        const int b = b0 + threadIdx.x;
        const size_t ri = ((size_t)BH + bh) * Rp + b;
        e0b_sh[threadIdx.x] = b < R ? p.mx_e0[ri] : 0;
        okb_sh[threadIdx.x] = b < R ? p.mx_ok[ri] : 0;
    }
    if (warp == 0) {
        tmem_alloc(&tmem_sh, kMxCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_sh;
    uint8_t* sA = sm;                               // parts h, m, l: 128 x D each
    uint8_t* sB = sm + kParts * kMxTile * D;        // parts h, m, l: 32 x D each
    bool issued = false;
    if (warp == 0) {
        mbar_expect_tx_w(&bar_ld, kParts * (kMxTile + kMxN) * D);
#pragma unroll
        for (int q = 0; q < kParts; ++q) {
            bulk_g2s_w(sA + q * kMxTile * D, qt + q * kMxTile * D, kMxTile * D, &bar_ld);
            bulk_g2s_w(sB + q * kMxN * D, kt + q * kMxTile * D + kslice, kMxN * D, &bar_ld);
        }
        if (__all_sync(0xffffffffu, mbar_wait(&bar_ld, 0, abort_v, p.status, p.wait_ns))) {
            tc_fence_after();
            // K-major no-swizzle: core matrices adjacent along K 128 bytes apart,
            // along the rows 8 D bytes apart; each MMA covers 32 channels (256 bytes)
            uint64_t dA[kParts], dB[kParts];
#pragma unroll
            for (int q = 0; q < kParts; ++q) {
                dA[q] = sdesc(sA + q * kMxTile * D, 128, 8 * D);
                dB[q] = sdesc(sB + q * kMxN * D, 128, 8 * D);
            }
            constexpr uint32_t id = idesc_i8(kMxTile, kMxN);
            // product (qa, qb) has weight 2^(7 (4 - qa - qb)) and goes to the
            // accumulator at column 32 (qa + qb); the first product issued into an
            // accumulator (the smallest qa of its sum) starts it
#pragma unroll
            for (int qa = 0; qa < kParts; ++qa)
#pragma unroll
                for (int qb = 0; qb < kParts; ++qb) {
                    const uint32_t acc_col = tmem + 32 * (qa + qb);
                    const int first_qa = qa + qb <= kParts - 1 ? 0 : qa + qb - (kParts - 1);
                    const bool first = qa == first_qa;
#pragma unroll
                    for (int kk = 0; kk < D / 32; ++kk)
                        mma_i8_w(acc_col, dA[qa] + 16 * kk, dB[qb] + 16 * kk, id, (first && kk == 0) ? 0u : 1u);
                }
            tc_commit_w(&bar_mma);
            issued = true;
        } else if (lane == 0 && !mbar_wait_drain(&bar_ld, 0, p.wait_ns)) {
            atomicOr(p.status, DA2_DEV_TIMEOUT);  // copies still in flight after the limit
        }
    }
    issued = __syncthreads_or(issued);
    const bool done = issued && mbar_wait(&bar_mma, 0, abort_v, p.status, p.wait_ns);
    tc_fence_after();
    // epilogue: thread = query block a (tensor-memory lane), 32 key blocks
    const int a = a0 + 32 * warp + lane;
    const size_t ra = (size_t)bh * Rp + a;
    const bool oka = a < R && p.mx_ok[ra];
    const int e0a = a < R ? p.mx_e0[ra] : 0;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * warp) << 16);
    if (__all_sync(0xffffffffu, done)) {
        // each warp stages its 32 rows x 32 columns in shared memory (rows
        // padded to 33 doubles against bank conflicts), then writes them row by
        // row, 32 consecutive key blocks per store
        double* stage = reinterpret_cast<double*>(sm + stage_off<D>()) + warp * 32 * 33;
#pragma unroll 1
        for (int c0 = 0; c0 < kMxN; c0 += 16) {
            uint32_t acc[kAcc][16];
#pragma unroll
            for (int q = 0; q < kAcc; ++q) tmem_ld16(lane_base + 32 * q + c0, acc[q]);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                long long T = 0;
#pragma unroll
                for (int q = 0; q < kAcc; ++q) T += (long long)(int)acc[q][j] << (7 * (kAcc - 1 - q));
                const int s = e0a + e0b_sh[c0 + j] - 14;  // within the normal range: |s| < 300
                const double scale = __longlong_as_double((long long)(s + 1023) << 52);
                stage[lane * 33 + c0 + j] = ((double)T * scale) * rd;
            }
        }
        __syncwarp();
        const int b = b0 + lane;
        const bool okc = b < R && okb_sh[lane];
#pragma unroll 4
        for (int r = 0; r < 32; ++r) {
            const int ar = a0 + 32 * warp + r;
            const bool okr = __shfl_sync(0xffffffffu, oka, r);
            if (okr && okc) p.Lmax[((size_t)bh * R + ar) * R + b] = stage[r * 33 + lane];
        }
    } else if (threadIdx.x == 0 && issued) {
        // the MMAs did not complete within the limit: wait for them before
        // the tensor memory is freed
        if (!mbar_wait_drain(&bar_mma, 0, p.wait_ns)) atomicOr(p.status, DA2_DEV_TIMEOUT);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, kMxCols);
}

// The fp64 chain for the blocks outside the exact range (the split kernel's
// list): for a flagged block r of side t, t = 0 recomputes row r of the head's
// max-pool logits (every key block), t = 1 column r (every query block).
template <int D>
__global__ void __launch_bounds__(128) mx_strips_kernel(PlanArgs p, double rd) {
    __shared__ double fixed[D];
    const int R = p.R, Rp = p.mx_rpad, BH = p.BH;
    const size_t plane = (size_t)BH * p.Rt * D;
    const int n = p.mx_fail[0];
    for (int i = blockIdx.x; i < n; i += gridDim.x) {
        const int ri = p.mx_fail[1 + i];
        const int r = ri % Rp, tb = ri / Rp, bh = tb % BH, t = tb / BH;
        const double* Q = p.desc + plane + (size_t)bh * p.Rt * D;      // max-pool Q descriptors
        const double* K = p.desc + 3 * plane + (size_t)bh * p.Rt * D;  // max-pool K descriptors
        const double* f = (t == 0 ? Q : K) + (size_t)r * D;
        __syncthreads();  // the previous strip's reads of fixed are done
        for (int c = threadIdx.x; c < D; c += 128) fixed[c] = f[c];
        __syncthreads();
        for (int o = threadIdx.x; o < R; o += 128) {
            const double* other = (t == 0 ? K : Q) + (size_t)o * D;
            double acc = 0.0;
            // q_c k_c in ascending c, as the logits kernel and the definition
            if (t == 0) {
#pragma unroll 8
                for (int c = 0; c < D; ++c) acc = fma(fixed[c], other[c], acc);
                p.Lmax[((size_t)bh * R + r) * R + o] = acc * rd;
            } else {
#pragma unroll 8
                for (int c = 0; c < D; ++c) acc = fma(other[c], fixed[c], acc);
                p.Lmax[((size_t)bh * R + o) * R + r] = acc * rd;
            }
        }
    }
}

}  // namespace

size_t mx_scratch_bytes(int BH, int R, int d) {
    const size_t Rp = (size_t)(R + kMxTile - 1) / kMxTile * kMxTile;
    size_t b = (size_t)2 * BH * Rp * kParts * d;  // the int8 parts of Q and K
    b = (b + 255) & ~(size_t)255;
    b += (size_t)2 * BH * Rp * sizeof(int);  // e0
    b = (b + 255) & ~(size_t)255;
    b += (size_t)2 * BH * Rp;  // row flags
    b = (b + 255) & ~(size_t)255;
    b += (1 + (size_t)2 * BH * Rp) * sizeof(int);  // list of the blocks outside the exact range
    return (b + 255) & ~(size_t)255;
}

void mx_carve(PlanArgs* p, char* c) {
    const int Rp = (p->R + kMxTile - 1) / kMxTile * kMxTile;
    p->mx_rpad = Rp;
    p->mx_tiles = reinterpret_cast<int8_t*>(c);
    size_t off = (size_t)2 * p->BH * Rp * kParts * p->d;
    off = (off + 255) & ~(size_t)255;
    p->mx_e0 = reinterpret_cast<int*>(c + off);
    off += (size_t)2 * p->BH * Rp * sizeof(int);
    off = (off + 255) & ~(size_t)255;
    p->mx_ok = reinterpret_cast<uint8_t*>(c + off);
    off += (size_t)2 * p->BH * Rp;
    off = (off + 255) & ~(size_t)255;
    p->mx_fail = reinterpret_cast<int*>(c + off);
}

cudaError_t launch_max_logits(const PlanArgs& p, double rd, cudaStream_t stream) {
    const int Rp = p.mx_rpad, BH = p.BH;
    cudaError_t e = cudaMemsetAsync(p.mx_fail, 0, sizeof(int), stream);
    if (e != cudaSuccess) return e;
    dim3 sg((Rp + 7) / 8, 2, BH);
    dim3 lg((p.R + kMxN - 1) / kMxN, Rp / kMxTile, BH);
    const int fg = 4 * (p.num_sms > 0 ? p.num_sms : 148);
    if (p.d == 64) {
        mx_split_kernel<64><<<sg, 256, 0, stream>>>(p);
        if ((e = cudaFuncSetAttribute(mx_logits_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMxSmem)) !=
            cudaSuccess)
            return e;
        mx_logits_kernel<64><<<lg, kMxThreads, kMxSmem, stream>>>(p, rd);
        mx_strips_kernel<64><<<fg, 128, 0, stream>>>(p, rd);
    } else {
        mx_split_kernel<128><<<sg, 256, 0, stream>>>(p);
        if ((e = cudaFuncSetAttribute(mx_logits_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, kMxSmem)) !=
            cudaSuccess)
            return e;
        mx_logits_kernel<128><<<lg, kMxThreads, kMxSmem, stream>>>(p, rd);
        mx_strips_kernel<128><<<fg, 128, 0, stream>>>(p, rd);
    }
    return cudaGetLastError();
}

}  // namespace da2

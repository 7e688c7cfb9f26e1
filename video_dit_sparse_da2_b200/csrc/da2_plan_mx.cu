// da2_plan_mx.cu -- the max-pool branch of the draft logits (DraftAttention2
// Eq. 3) from exact integer tensor-core products.
//
// The draft defines a logit as an fp64 fma chain over the channels in
// ascending order, times 1/sqrt(d).  The max-pool descriptors are channel
// maxima of bf16 inputs, so every one of them is a bf16 value: sign, 8-bit
// significand M (with its leading bit) and exponent E.  Within a block (one
// row of the descriptor matrix) whose nonzero values span at most kMaxSpan
// binades above the smallest exponent e0, every value is N * 2^(e0 - 7) with
// an integer |N| < 2^14.  The product of two rows is then
// T * 2^(e0_a + e0_b - 14) with T = sum_c N_ac N_bc, |T| < 2^35; every partial
// sum of the defining fp64 chain is such an integer multiple below 2^53 units,
// so the chain is exact and equals T * 2^(...) exactly.  T itself is computed
// exactly by 8-bit tensor-core MMAs (tcgen05.mma kind::i8, s32 accumulation)
// on the split N = 128 hi + lo (hi in [-128, 127], lo in [0, 127]):
//   T = 2^14 sum hi hi' + 2^7 (sum hi lo' + sum lo hi') + sum lo lo'.
// The logit is then (double)T * 2^(e0_a + e0_b - 14) (exact) * (1/sqrt d)
// (one rounding): bit for bit the defining value.  A block outside that range
// (or holding a value that is not a bf16 value) is marked, and the fp64 chain
// of the logits kernel computes every pair that involves it.
#include "da2_common.cuh"
#include "da2_kernels.h"

namespace da2 {

namespace {

constexpr int kMaxSpan = 6;      // binades above e0: |N| <= 255 * 2^6 < 2^14
constexpr int kMxTile = 128;     // rows per split tile (the MMA's M)
constexpr int kMxN = 64;         // key blocks per MMA tile (the MMA's N)
constexpr uint32_t kMxCols = 256;  // tensor-memory columns: HH, HL + LH, LL (3 x 64 used)
constexpr int kMxThreads = 128;
// dynamic shared memory: hi / lo tiles of A (128 rows) and B (64 rows), then
// the epilogue's staging rows (4 warps x 32 x 33 doubles)
template <int D>
constexpr int stage_off() { return 384 * D; }
constexpr int kStageBytes = 4 * 32 * 33 * 8;

__device__ __forceinline__ uint32_t kmajor_off_b(int row, int byte, int row_bytes) {
    return ((row >> 3) * (row_bytes >> 4) + (byte >> 4)) * 128 + (row & 7) * 16 + (byte & 15);
}

// One warp per descriptor row (block r of head bh, tensor t: 0 = Q max, 1 = K
// max): lane l handles channels 4l .. 4l+3.  Writes the hi / lo int8 tiles in
// the tcgen05 K-major no-swizzle layout (128-row tiles), e0 and the row flag,
// and clears the tile flag of a tile that holds a row outside the exact range.
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
    uint32_t hi4 = 0u, lo4 = 0u;
    if (ok) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int N = nz[i] ? m[i] * (1 << (e[i] - e0)) : 0;
            const int h = N >> 7;  // floor: N = 128 h + lo, lo in [0, 127]
            const int l = N - 128 * h;
            hi4 |= ((uint32_t)h & 0xFFu) << (8 * i);
            lo4 |= (uint32_t)l << (8 * i);
        }
    }
    // tiles [2][BH][Rp/128][hi, lo][128 * D]
    const size_t tile = ((size_t)t * p.BH + bh) * (Rp / kMxTile) + r / kMxTile;
    int8_t* hi = p.mx_tiles + tile * 2 * kMxTile * D;
    int8_t* lo = hi + kMxTile * D;
    if (lane < kLanes) {
        const uint32_t o = kmajor_off_b(r % kMxTile, 4 * lane, D);
        *reinterpret_cast<uint32_t*>(hi + o) = hi4;
        *reinterpret_cast<uint32_t*>(lo + o) = lo4;
    }
    if (lane == 0) {
        const size_t ri = ((size_t)t * p.BH + bh) * Rp + r;
        p.mx_e0[ri] = e0;
        p.mx_ok[ri] = ok ? 1 : 0;
        if (!ok) p.mx_tile_ok[((size_t)t * p.BH + bh) * (Rp / kMxTile) + r / kMxTile] = 0;
    }
}

// One CTA per (head, 128 query blocks, 64 key blocks): T of every pair from
// four int8 products, then the logit; pairs whose query or key block is
// outside the exact range are left to the fp64 chain.
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
    const int8_t* qt = p.mx_tiles + ((size_t)bh * ntile + at) * 2 * kMxTile * D;                 // Q hi, lo
    const int8_t* kt = p.mx_tiles + (((size_t)BH + bh) * ntile + b0 / kMxTile) * 2 * kMxTile * D;  // K hi, lo
    const size_t kslice = (size_t)(b0 % kMxTile) * D;  // rows b0 % 128 .. +63 of the K tile
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
    uint8_t* sAh = sm;
    uint8_t* sAl = sm + kMxTile * D;
    uint8_t* sBh = sm + 2 * kMxTile * D;
    uint8_t* sBl = sBh + kMxN * D;
    bool issued = false;
    if (warp == 0) {
        mbar_expect_tx_w(&bar_ld, 2 * kMxTile * D + 2 * kMxN * D);
        bulk_g2s_w(sAh, qt, kMxTile * D, &bar_ld);
        bulk_g2s_w(sAl, qt + kMxTile * D, kMxTile * D, &bar_ld);
        bulk_g2s_w(sBh, kt + kslice, kMxN * D, &bar_ld);
        bulk_g2s_w(sBl, kt + kMxTile * D + kslice, kMxN * D, &bar_ld);
        if (__all_sync(0xffffffffu, mbar_wait(&bar_ld, 0, abort_v, p.status, p.wait_ns))) {
            tc_fence_after();
            // K-major no-swizzle: core matrices adjacent along K 128 bytes apart,
            // along the rows 8 D bytes apart; each MMA covers 32 channels (256 bytes)
            const uint64_t dAh = sdesc(sAh, 128, 8 * D), dAl = sdesc(sAl, 128, 8 * D);
            const uint64_t dBh = sdesc(sBh, 128, 8 * D), dBl = sdesc(sBl, 128, 8 * D);
            constexpr uint32_t id = idesc_i8(kMxTile, kMxN);
#pragma unroll
            for (int kk = 0; kk < D / 32; ++kk) mma_i8_w(tmem, dAh + 16 * kk, dBh + 16 * kk, id, kk > 0);
#pragma unroll
            for (int kk = 0; kk < D / 32; ++kk) mma_i8_w(tmem + 64, dAh + 16 * kk, dBl + 16 * kk, id, kk > 0);
#pragma unroll
            for (int kk = 0; kk < D / 32; ++kk) mma_i8_w(tmem + 64, dAl + 16 * kk, dBh + 16 * kk, id, 1u);
#pragma unroll
            for (int kk = 0; kk < D / 32; ++kk) mma_i8_w(tmem + 128, dAl + 16 * kk, dBl + 16 * kk, id, kk > 0);
            tc_commit_w(&bar_mma);
            issued = true;
        } else if (lane == 0 && !mbar_wait_drain(&bar_ld, 0, p.wait_ns)) {
            atomicOr(p.status, DA2_DEV_TIMEOUT);  // copies still in flight after the limit
        }
    }
    __syncthreads();
    issued = __syncthreads_or(issued);
    const bool done = issued && mbar_wait(&bar_mma, 0, abort_v, p.status, p.wait_ns);
    tc_fence_after();
    // epilogue: thread = query block a (tensor-memory lane), 64 key blocks
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
        for (int c0 = 0; c0 < kMxN; c0 += 32) {
            uint32_t hh[32], hx[32], ll[32];
            tmem_ld32(lane_base + c0, hh);
            tmem_ld32(lane_base + 64 + c0, hx);
            tmem_ld32(lane_base + 128 + c0, ll);
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const long long T = ((long long)(int)hh[j] << 14) + ((long long)(int)hx[j] << 7) + (long long)(int)ll[j];
                const int s = e0a + e0b_sh[c0 + j] - 14;  // within the normal range: |s| < 300
                const double scale = __longlong_as_double((long long)(s + 1023) << 52);
                stage[lane * 33 + j] = ((double)T * scale) * rd;
            }
            __syncwarp();
            const int b = b0 + c0 + lane;
            const bool okc = b < R && okb_sh[c0 + lane];
#pragma unroll 4
            for (int r = 0; r < 32; ++r) {
                const int ar = a0 + 32 * warp + r;
                const bool okr = __shfl_sync(0xffffffffu, oka, r);
                if (okr && okc) p.Lmax[((size_t)bh * R + ar) * R + b] = stage[r * 33 + lane];
            }
            __syncwarp();
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

}  // namespace

size_t mx_scratch_bytes(int BH, int R, int d) {
    const size_t Rp = (size_t)(R + kMxTile - 1) / kMxTile * kMxTile;
    size_t b = (size_t)2 * BH * Rp * 2 * d;  // hi and lo tiles of Q and K
    b = (b + 255) & ~(size_t)255;
    b += (size_t)2 * BH * Rp * sizeof(int);  // e0
    b = (b + 255) & ~(size_t)255;
    b += (size_t)2 * BH * Rp;  // row flags
    b = (b + 255) & ~(size_t)255;
    b += (size_t)2 * BH * (Rp / kMxTile);  // tile flags
    return (b + 255) & ~(size_t)255;
}

void mx_carve(PlanArgs* p, char* c) {
    const int Rp = (p->R + kMxTile - 1) / kMxTile * kMxTile;
    p->mx_rpad = Rp;
    p->mx_tiles = reinterpret_cast<int8_t*>(c);
    size_t off = (size_t)2 * p->BH * Rp * 2 * p->d;
    off = (off + 255) & ~(size_t)255;
    p->mx_e0 = reinterpret_cast<int*>(c + off);
    off += (size_t)2 * p->BH * Rp * sizeof(int);
    off = (off + 255) & ~(size_t)255;
    p->mx_ok = reinterpret_cast<uint8_t*>(c + off);
    off += (size_t)2 * p->BH * Rp;
    off = (off + 255) & ~(size_t)255;
    p->mx_tile_ok = reinterpret_cast<uint8_t*>(c + off);
}

int mx_tile_rows() { return kMxTile; }

cudaError_t launch_max_logits(const PlanArgs& p, double rd, cudaStream_t stream) {
    const int Rp = p.mx_rpad, BH = p.BH;
    cudaError_t e = cudaMemsetAsync(p.mx_tile_ok, 1, (size_t)2 * BH * (Rp / kMxTile), stream);
    if (e != cudaSuccess) return e;
    dim3 sg((Rp + 7) / 8, 2, BH);
    dim3 lg((p.R + kMxN - 1) / kMxN, Rp / kMxTile, BH);
    // 84 KB per CTA: the tiles and the epilogue's staging rows, and more than a
    // third of the multiprocessor's shared memory, so that no more than two
    // CTAs (2 x 256 of the 512 tensor-memory columns) share a multiprocessor
    static_assert(384 * 128 + kStageBytes <= 84 * 1024, "tiles and staging fit");
    const int smem = 84 * 1024;
    if (p.d == 64) {
        mx_split_kernel<64><<<sg, 256, 0, stream>>>(p);
        if ((e = cudaFuncSetAttribute(mx_logits_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) !=
            cudaSuccess)
            return e;
        mx_logits_kernel<64><<<lg, kMxThreads, smem, stream>>>(p, rd);
    } else {
        mx_split_kernel<128><<<sg, 256, 0, stream>>>(p);
        if ((e = cudaFuncSetAttribute(mx_logits_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) !=
            cudaSuccess)
            return e;
        mx_logits_kernel<128><<<lg, kMxThreads, smem, stream>>>(p, rd);
    }
    return cudaGetLastError();
}

}  // namespace da2

// da2_plan.cu -- draft map and routing ("DraftAttention2", Eq. 3; Sec. 3.1
// "Joint allocation of sparsity and precision"; App. C.1 "Routing and
// precision formats").
//
// The ranking of all R^2 region pairs of a head must be reproducible bit for
// bit, so the draft map is computed in fp64 with a fixed operation order:
//   logit(a,b) = (fma chain over channels c = 0..d-1 in ascending order,
//                 starting from 0) * (1/sqrt d)
//   per row and branch: m = max_b logit; e_b = exp_fixed(logit_b - m);
//                 Z = sum of e_b in ascending b; S_b = e_b / Z
//   A = fma(lambda, S^max, (1 - lambda) * S^avg)
// exp_fixed is a Cody-Waite reduction with a two-part ln2 and a degree-13
// Taylor polynomial in Horner form (fma), scaled by 2^k; results below the
// normal range are flushed to zero.  The ranking is an exact radix selection
// of the C16-th, C8-th and Ck-th largest 96-bit keys (A bits : ~pair index)
// -- the cumulative cuts of the 16-bit, 8-bit and kept tiers --, i.e.
// A descending with ties to the smaller pair index a*R+b, followed by an
// exact classification, a scan of the rows' counts into list offsets and an
// ordered compaction of every row's list at its offset.
#include <algorithm>
#include <cfloat>

#include "da2_common.cuh"
#include "da2_kernels.h"

namespace da2 {

namespace {

constexpr double kLog2e = 0x1.71547652b82fep+0;   // 1/ln 2
constexpr double kLn2Hi = 0x1.62e42fee00000p-1;   // ln 2 cut to 32 significant bits
constexpr double kLn2Lo = 0x1.a39ef35793c76p-33;  // ln 2 - kLn2Hi
// 1/n! for n = 0..13, correctly rounded
__constant__ double kInvFact[14] = {
    0x1.0000000000000p+0,  0x1.0000000000000p+0,  0x1.0000000000000p-1,  0x1.5555555555555p-3,
    0x1.5555555555555p-5,  0x1.1111111111111p-7,  0x1.6c16c16c16c17p-10, 0x1.a01a01a01a01ap-13,
    0x1.a01a01a01a01ap-16, 0x1.71de3a556c734p-19, 0x1.27e4fb7789f5cp-22, 0x1.ae64567f544e4p-26,
    0x1.1eed8eff8d898p-29, 0x1.6124613a86d09p-33};

__device__ __forceinline__ double exp_fixed(double x) {
    if (x < -708.0) return 0.0;
    if (x > 709.0) return __longlong_as_double(0x7ff0000000000000LL);
    const double k = rint(x * kLog2e);
    double r = fma(-k, kLn2Hi, x);
    r = fma(-k, kLn2Lo, r);
    double p = kInvFact[13];
#pragma unroll
    for (int n = 12; n >= 0; --n) p = fma(p, r, kInvFact[n]);
    // 2^k with k in [-1021, 1023]: the product is a normal number, exact.
    return p * __longlong_as_double((long long)((int)k + 1023) << 52);
}

// ---------------------------------------------------------------- logits
// One branch (average or max descriptors) of one head per CTA, 128 x 128
// output tile; each thread owns 8 x 8 outputs: rows {2ty, 2ty+1} + 32 i and
// columns {2tx, 2tx+1} + 32 j (i, j < 4), so that the 16-byte shared-memory
// reads of a warp are contiguous.  Channels are staged 16 at a time
// (transposed, [channel][row]) in two shared buffers; every output is one fma
// chain over c = 0..d-1 in ascending order starting from 0, as defined.
constexpr int kLgTile = 128, kLgKc = 16, kLgThreads = 256;
constexpr size_t kLgSmem = 2ull * 2 * kLgKc * kLgTile * sizeof(double);  // 64 KB

template <int D>
__global__ void __launch_bounds__(kLgThreads, 1) logits_kernel(PlanArgs p, double rd) {
    extern __shared__ __align__(16) double lg_smem[];
    double* sQ = lg_smem;                          // [2][kLgKc][kLgTile]
    double* sK = lg_smem + 2 * kLgKc * kLgTile;    // [2][kLgKc][kLgTile]
    const int R = p.R, bh = blockIdx.z >> 1, branch = blockIdx.z & 1;
    const int a0 = blockIdx.y * kLgTile, b0 = blockIdx.x * kLgTile;
    // the max-pool branch comes from the exact integer tensor-core path and
    // its fp64 strips (launch_max_logits)
    if (branch == 1) return;
    const int t = threadIdx.x, tx = t & 15, ty = t >> 4;
    // descriptors of every block are stored (Rt per head); the draft uses the
    // R video blocks
    const size_t plane = (size_t)p.BH * p.Rt * D;
    const double* Qs = p.desc + (size_t)branch * plane + (size_t)bh * p.Rt * D;
    const double* Ks = p.desc + (size_t)(2 + branch) * plane + (size_t)bh * p.Rt * D;

    // staging: thread t moves channel pairs of rows (t + 256 it) % 128
    double2 rq[4], rk[4];
    auto fetch = [&](int k0) {
#pragma unroll
        for (int it = 0; it < 4; ++it) {
            const int idx = it * kLgThreads + t, row = idx & (kLgTile - 1), cp = idx >> 7;
            const int ra = a0 + row, rb = b0 + row;
            rq[it] = ra < R ? *reinterpret_cast<const double2*>(Qs + (size_t)ra * D + k0 + 2 * cp)
                            : make_double2(0.0, 0.0);
            rk[it] = rb < R ? *reinterpret_cast<const double2*>(Ks + (size_t)rb * D + k0 + 2 * cp)
                            : make_double2(0.0, 0.0);
        }
    };
    auto stage = [&](int buf) {
        double* q = sQ + buf * kLgKc * kLgTile;
        double* k = sK + buf * kLgKc * kLgTile;
#pragma unroll
        for (int it = 0; it < 4; ++it) {
            const int idx = it * kLgThreads + t, row = idx & (kLgTile - 1), cp = idx >> 7;
            q[(2 * cp) * kLgTile + row] = rq[it].x;
            q[(2 * cp + 1) * kLgTile + row] = rq[it].y;
            k[(2 * cp) * kLgTile + row] = rk[it].x;
            k[(2 * cp + 1) * kLgTile + row] = rk[it].y;
        }
    };

    double acc[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.0;

    fetch(0);
    stage(0);
    __syncthreads();
    constexpr int NCH = D / kLgKc;
#pragma unroll 1
    for (int ch = 0; ch < NCH; ++ch) {
        const int buf = ch & 1;
        if (ch + 1 < NCH) fetch((ch + 1) * kLgKc);  // global loads in flight during the FMAs
        const double* q = sQ + buf * kLgKc * kLgTile;
        const double* k = sK + buf * kLgKc * kLgTile;
#pragma unroll
        for (int c = 0; c < kLgKc; ++c) {
            double qa[8], kb[8];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const double2 x = *reinterpret_cast<const double2*>(q + c * kLgTile + 32 * i + 2 * ty);
                const double2 y = *reinterpret_cast<const double2*>(k + c * kLgTile + 32 * i + 2 * tx);
                qa[2 * i] = x.x;
                qa[2 * i + 1] = x.y;
                kb[2 * i] = y.x;
                kb[2 * i + 1] = y.y;
            }
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[i][j] = fma(qa[i], kb[j], acc[i][j]);
        }
        if (ch + 1 < NCH) {
            stage(buf ^ 1);  // the other buffer was last read before the previous barrier
            __syncthreads();
        }
    }
    double* out = branch ? p.Lmax : p.A;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int a = a0 + 32 * (i >> 1) + 2 * ty + (i & 1);
        if (a >= R) continue;
        double* orow = out + ((size_t)bh * R + a) * R;
#pragma unroll
        for (int j = 0; j < 8; j += 2) {
            const int b = b0 + 32 * (j >> 1) + 2 * tx;
            if (b + 1 < R && ((R & 1) == 0)) {
                *reinterpret_cast<double2*>(orow + b) = make_double2(acc[i][j] * rd, acc[i][j + 1] * rd);
            } else {
                if (b < R) orow[b] = acc[i][j] * rd;
                if (b + 1 < R) orow[b + 1] = acc[i][j + 1] * rd;
            }
        }
    }
}

// ---------------------------------------------------------------- softmax
// One CTA per (head, query region): both branches, fixed summation order.
constexpr int kSoftThreads = 128;

__device__ __forceinline__ double block_max(double v, double* red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    double m = red[0];
#pragma unroll
    for (int w = 1; w < kSoftThreads / 32; ++w) m = fmax(m, red[w]);
    __syncthreads();
    return m;
}

__global__ void __launch_bounds__(kSoftThreads) softmax_kernel(PlanArgs p) {
    extern __shared__ double sm[];
    __shared__ double red[kSoftThreads / 32];
    __shared__ double Z[2];
    __shared__ unsigned long long mm[2][kSoftThreads / 32];
    const int R = p.R;
    const size_t row = blockIdx.x;
    const int bh = (int)(row / R);
    double* la = sm;
    double* lm = sm + R;
    double* Arow = p.A + row * R;
    const double* Mrow = p.Lmax + row * R;
    double ma = -DBL_MAX, mx = -DBL_MAX;
    for (int b = threadIdx.x; b < R; b += kSoftThreads) {
        const double x = Arow[b], y = Mrow[b];
        la[b] = x;
        lm[b] = y;
        ma = fmax(ma, x);
        mx = fmax(mx, y);
    }
    ma = block_max(ma, red);
    mx = block_max(mx, red);
    for (int b = threadIdx.x; b < R; b += kSoftThreads) {
        la[b] = exp_fixed(la[b] - ma);
        lm[b] = exp_fixed(lm[b] - mx);
    }
    __syncthreads();
    if (threadIdx.x == 0 || threadIdx.x == 32) {
        const double* e = threadIdx.x == 0 ? la : lm;
        double z = 0.0;
        for (int b = 0; b < R; ++b) z += e[b];
        Z[threadIdx.x == 0 ? 0 : 1] = z;
    }
    __syncthreads();
    const double za = Z[0], zm = Z[1];
    const double lam = p.lambda, oml = 1.0 - p.lambda;
    unsigned long long lo = ~0ull, hi = 0ull;
    for (int b = threadIdx.x; b < R; b += kSoftThreads) {
        const double A = fma(lam, lm[b] / zm, oml * (la[b] / za));
        Arow[b] = A;
        const unsigned long long bits = (unsigned long long)__double_as_longlong(A);
        lo = bits < lo ? bits : lo;
        hi = bits > hi ? bits : hi;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const unsigned long long l2 = __shfl_xor_sync(0xffffffffu, lo, o);
        const unsigned long long h2 = __shfl_xor_sync(0xffffffffu, hi, o);
        lo = l2 < lo ? l2 : lo;
        hi = h2 > hi ? h2 : hi;
    }
    if ((threadIdx.x & 31) == 0) {
        mm[0][threadIdx.x >> 5] = lo;
        mm[1][threadIdx.x >> 5] = hi;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < kSoftThreads / 32; ++w) {
            lo = mm[0][w] < lo ? mm[0][w] : lo;
            hi = mm[1][w] > hi ? mm[1][w] : hi;
        }
        atomicMin(&p.abits_minmax[bh], lo);
        atomicMax(&p.abits_minmax[p.BH + bh], hi);
    }
}

// ---------------------------------------------------------------- selection
// Key of pair i of a head: 96 bits = A bits (64) : 0xFFFFFFFF - i (32).
// Larger key = higher rank (larger A, or equal A and smaller index).
struct Key {
    unsigned long long hi;
    unsigned int lo;
};

constexpr int kTargets = 3;  // selection targets per head (16-bit, 8-bit, kept cuts)
// Keys a head's candidate list holds at most: the first pass in which the open
// targets' prefixes match at most this many keys in all collects them, and the
// later passes read the list instead of the whole draft map.  The list (A bits,
// then ~pair index) sits in the head's rows of the max-branch logits, which the
// softmax kernel has consumed: R^2 doubles hold min(kSelectCand, 2 R^2 / 3) keys.
constexpr int kSelectCand = 16384;
__host__ __device__ inline int select_cand_cap(int R) {
    const long long c = 2ll * R * R / 3;
    return c < kSelectCand ? (int)c : kSelectCand;
}

__device__ __forceinline__ void top_mask(int nbits, unsigned long long* mh, unsigned int* ml) {
    *mh = nbits <= 0 ? 0ull : (nbits >= 64 ? ~0ull : (~0ull << (64 - nbits)));
    const int nl = nbits - 64;
    *ml = nl <= 0 ? 0u : (nl >= 32 ? ~0u : (~0u << (32 - nl)));
}

__device__ __forceinline__ unsigned digit_at(Key k, int pos, int w) {
    // bits [pos, pos + w) of the 96-bit key, bit 0 = lsb of lo
    const unsigned mask = (1u << w) - 1u;
    if (pos >= 32) return (unsigned)(k.hi >> (pos - 32)) & mask;
    if (pos + w <= 32) return (k.lo >> pos) & mask;
    return (unsigned)((k.hi << (32 - pos)) | (unsigned long long)(k.lo >> pos)) & mask;
}

// Targets of a head, in order: the C16-th, C8-th and Ck-th largest keys (the
// cumulative cuts of the 16-bit, 8-bit and kept tiers); a cut of 0 is "none".
__global__ void select_init_kernel(PlanArgs p, long long C16, long long C8, long long Ck) {
    const int bh = blockIdx.x * blockDim.x + threadIdx.x;
    if (bh >= p.BH) return;
    const unsigned long long lo = p.abits_minmax[bh], hi = p.abits_minmax[p.BH + bh];
    const int c = (lo == hi) ? 64 : __clzll((long long)(lo ^ hi));
    for (int t = 0; t < kTargets; ++t) {
        SelectTarget s;
        s.nbits = c;
        s.p_hi = (c >= 64) ? lo : (c == 0 ? 0ull : (lo & (~0ull << (64 - c))));
        s.p_lo = 0u;
        s.need = t == 0 ? C16 : (t == 1 ? C8 : Ck);
        s.unique = 0;
        s.found = 0;
        s.matches = (long long)p.R * p.R;
        s.none = s.need == 0;
        s.done = s.none;
        s.key_hi = 0ull;
        s.key_lo = 0u;
        p.sel[bh * kTargets + t] = s;
    }
    p.cand_n[bh] = 0;
    p.cand_state[bh] = 0;
}

constexpr int kHistThreads = 1024;
constexpr int kHistMinChunk = 16384;             // keys per CTA at least (16 per thread)
constexpr long long kHistDirect = 1ll << 14;     // at most this many matching keys: count in global memory

// Choose the digit that holds the sought rank of target t of head bh (one
// warp), from the completed histogram of the pass, and clear the histogram.
__device__ void select_scan_warp(PlanArgs& p, int bh, int t, int lane) {
    unsigned* gh = p.hist + ((size_t)bh * kTargets + t) * 4096;
    SelectTarget* sp = &p.sel[bh * kTargets + t];
    // from L2: another CTA of this pass may have recorded the unique key
    SelectTarget s;
    static_assert(sizeof(SelectTarget) % 16 == 0, "SelectTarget is read as 16-byte words");
#pragma unroll
    for (int i = 0; i < (int)(sizeof(SelectTarget) / 16); ++i)
        reinterpret_cast<uint4*>(&s)[i] = __ldcg(reinterpret_cast<const uint4*>(sp) + i);
    if (!s.done && s.unique) {
        if (s.found) {
            s.done = 1;
            if (lane == 0) *sp = s;
        }
    } else if (!s.done) {
        const int w = min(12, 96 - s.nbits), pos = 96 - s.nbits - w;
        // lane covers bins [4095 - 128 lane - 127, 4095 - 128 lane], descending
        const int top = 4095 - 128 * lane;
        unsigned long long sum = 0;
        for (int i = 0; i < 128; ++i) sum += __ldcg(&gh[top - i]);
        unsigned long long incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned long long v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        const unsigned long long excl = incl - sum;
        const bool mine = (long long)excl < s.need && s.need <= (long long)incl;
        if (mine) {
            long long cum = (long long)excl;
            for (int i = 0; i < 128; ++i) {
                const int bin = top - i;
                const long long c = __ldcg(&gh[bin]);
                if (cum + c >= s.need) {
                    s.need -= cum;
                    if (pos >= 32) s.p_hi |= (unsigned long long)bin << (pos - 32);
                    else {
                        s.p_lo |= (unsigned)bin << pos;
                        if (pos + w > 32) s.p_hi |= (unsigned long long)bin >> (32 - pos);
                    }
                    s.nbits += w;
                    s.matches = c;
                    if (s.nbits >= 96) {
                        s.done = 1;
                        s.key_hi = s.p_hi;
                        s.key_lo = s.p_lo;
                    } else if (c == 1) {
                        s.unique = 1;
                    }
                    *sp = s;
                    break;
                }
                cum += c;
            }
        }
    }
    __syncwarp();
    for (int i = lane; i < 4096; i += 32) gh[i] = 0u;
}

// One pass of the radix selection: histogram of the next digit of the keys
// that match each target's prefix; the last CTA of a head to finish chooses
// the digits (select_scan_warp).  A target whose prefix matches one key
// records that key here and is marked done by that pass's scan, so the
// `done` flags do not change while a pass runs.
template <int NT>
__global__ void __launch_bounds__(kHistThreads) select_hist_kernel(PlanArgs p, int chunk) {
    extern __shared__ unsigned h_dyn[];  // [NT][4096]
    __shared__ int is_last;
    constexpr int t0 = kTargets - NT;     // with no 16-bit tier only the last two targets are live
    const int bh = blockIdx.y, tid = threadIdx.x;
    SelectTarget s[NT];
    bool all_done = true;
#pragma unroll
    for (int t = 0; t < NT; ++t) {
        s[t] = p.sel[bh * kTargets + t0 + t];
        all_done = all_done && s[t].done;
    }
    if (all_done) return;
    bool in_smem[NT], any_smem = false;
#pragma unroll
    for (int t = 0; t < NT; ++t) {
        in_smem[t] = !s[t].done && !s[t].unique && s[t].matches > kHistDirect;
        any_smem = any_smem || in_smem[t];
    }
    if (any_smem) {
        for (int i = tid; i < NT * 4096; i += kHistThreads) h_dyn[i] = 0u;
        __syncthreads();
    }
    unsigned long long mh[NT];
    unsigned ml[NT];
    int w[NT], pos[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) {
        top_mask(s[t].nbits, &mh[t], &ml[t]);
        w[t] = min(12, 96 - s[t].nbits);
        pos[t] = 96 - s[t].nbits - w[t];
    }
    unsigned* gh = p.hist + ((size_t)bh * kTargets + t0) * 4096;
    const size_t RR = (size_t)p.R * p.R;
    const size_t begin = (size_t)blockIdx.x * chunk;
    const double* Ah = p.A + (size_t)bh * RR;
    // candidate list: read it once collected; collect it in the first pass in
    // which the open targets match at most kSelectCand keys together (a key
    // matching any open prefix is kept: the prefixes only grow from here)
    long long live = 0;
#pragma unroll
    for (int t = 0; t < NT; ++t)
        if (!s[t].done) live += s[t].unique ? 1 : s[t].matches;
    const int cap = select_cand_cap(p.R);
    const int cstate = p.cand_state[bh];
    const bool from_list = cstate == 1, collect = cstate == 0 && live <= cap;
    unsigned long long* ch = reinterpret_cast<unsigned long long*>(p.Lmax + (size_t)bh * RR);
    unsigned* cl = reinterpret_cast<unsigned*>(ch + cap);
    // histogram (or record) key k for every open target whose prefix it
    // matches; true when it matches one
    auto count_key = [&](Key k) -> bool {
        bool any = false;
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            if (s[t].done) continue;
            if (((k.hi ^ s[t].p_hi) & mh[t]) || ((k.lo ^ s[t].p_lo) & ml[t])) continue;
            any = true;
            if (s[t].unique) {
                p.sel[bh * kTargets + t0 + t].key_hi = k.hi;
                p.sel[bh * kTargets + t0 + t].key_lo = k.lo;
                p.sel[bh * kTargets + t0 + t].found = 1;
            } else if (in_smem[t]) {
                atomicAdd(&h_dyn[t * 4096 + digit_at(k, pos[t], w[t])], 1u);
            } else {
                atomicAdd(&gh[t * 4096 + digit_at(k, pos[t], w[t])], 1u);
            }
        }
        return any;
    };
    auto count = [&](size_t i, double a) {
        Key k;
        k.hi = (unsigned long long)__double_as_longlong(a);
        k.lo = 0xFFFFFFFFu - (unsigned)i;
        if (count_key(k) && collect) {
            // at most `live` keys match an open prefix, so the list cannot overflow
            const int slot = atomicAdd(&p.cand_n[bh], 1);
            if (slot < cap) {
                ch[slot] = k.hi;
                cl[slot] = k.lo;
            }
        }
    };
    if (from_list) {
        // the keys still in play were collected by an earlier pass: the first
        // CTA of the head goes through them, the others only report
        if (blockIdx.x == 0) {
            const int n = min(__ldcg(&p.cand_n[bh]), cap);
            for (int i = tid; i < n; i += kHistThreads) {
                Key k;
                k.hi = __ldcg(&ch[i]);
                k.lo = __ldcg(&cl[i]);
                count_key(k);
            }
        }
    } else {
        // chunk / kHistThreads keys per thread (a multiple of 4), four loads in flight
#pragma unroll 1
        for (int k0 = 0; k0 < chunk / kHistThreads; k0 += 4) {
            double a[4];
            size_t idx[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                idx[u] = begin + (size_t)(k0 + u) * kHistThreads + tid;
                a[u] = idx[u] < RR ? __ldcs(Ah + idx[u]) : 0.0;
            }
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (idx[u] < RR) count(idx[u], a[u]);
        }
    }
    if (any_smem) {
        __syncthreads();
        for (int i = tid; i < NT * 4096; i += kHistThreads) {
            const unsigned v = h_dyn[i];
            if (v) atomicAdd(&gh[i], v);
        }
    }
    // the last CTA of this head to finish chooses the digits
    __threadfence();
    __syncthreads();
    if (tid == 0) is_last = atomicAdd(&p.done_count[bh], 1u) == gridDim.x - 1;
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    if (tid < 32 * NT) select_scan_warp(p, bh, t0 + (tid >> 5), tid & 31);
    if (tid == 0) {
        p.done_count[bh] = 0u;
        if (collect) p.cand_state[bh] = 1;  // every CTA of the head has appended its keys
    }
}

// ---------------------------------------------------------------- classify
// One warp per (head, query region): precision of every pair (16, 8, 4 or 0)
// and the row's numbers of 8-bit, 4-bit and 16-bit key blocks.
__global__ void __launch_bounds__(128) classify_kernel(PlanArgs p) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const size_t row = (size_t)blockIdx.x * 4 + warp;
    const int R = p.R;
    if (row >= (size_t)p.BH * R) return;
    const int bh = (int)(row / R), a = (int)(row % R);
    const SelectTarget s16 = p.sel[bh * kTargets], s8 = p.sel[bh * kTargets + 1], sk = p.sel[bh * kTargets + 2];
    const double* Arow = p.A + row * R;
    uint8_t* prow = p.prec + row * R;
    auto ge = [](Key k, const SelectTarget& s) {
        return !s.none && (k.hi > s.key_hi || (k.hi == s.key_hi && k.lo >= s.key_lo));
    };
    int n16 = 0, n8 = 0, n4 = 0;
    for (int b0 = 0; b0 < R; b0 += 32) {
        const int b = b0 + lane;
        bool is16 = false, is8 = false, is4 = false;
        if (b < R) {
            Key k;
            k.hi = (unsigned long long)__double_as_longlong(Arow[b]);
            k.lo = 0xFFFFFFFFu - (unsigned)(a * R + b);
            is16 = ge(k, s16);
            is8 = !is16 && ge(k, s8);
            is4 = !is16 && !is8 && ge(k, sk);
            prow[b] = is16 ? 16 : (is8 ? 8 : (is4 ? 4 : 0));
        }
        n16 += __popc(__ballot_sync(0xffffffffu, is16));
        n8 += __popc(__ballot_sync(0xffffffffu, is8));
        n4 += __popc(__ballot_sync(0xffffffffu, is4));
    }
    if (lane == 0) {
        const size_t BHRt = (size_t)p.BH * p.Rt, rt = (size_t)bh * p.Rt + a;
        p.cnt[rt] = n8;
        p.cnt[BHRt + rt] = n4;
        p.cnt[2 * BHRt + rt] = n16 + p.Rp;  // every prefix key is kept at 16 bits
    }
}

// ---------------------------------------------------------------- lists
// Compact lists: row a of head bh owns kidx[off[bh][a] .. off[bh][a+1]).
// The kept pairs of a head number exactly `per_head` (the quota), so head bh
// starts at bh * per_head; one warp per head scans its rows' counts.
__global__ void offsets_kernel(PlanArgs p, long long per_head) {
    const int bh = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (bh >= p.BH) return;
    const int Rt = p.Rt;
    const size_t BHRt = (size_t)p.BH * Rt;
    long long base = (long long)bh * per_head;
    long long* off = p.off + (size_t)bh * (Rt + 1);
    for (int a0 = 0; a0 < Rt; a0 += 32) {
        const int a = a0 + lane;
        const size_t row = (size_t)bh * Rt + a;
        // a prefix row keeps every block at 16 bits (non-sparse, App. C.1)
        const long long n = a >= Rt ? 0 : (a >= p.R ? (long long)Rt
                                                     : (long long)p.cnt[row] + p.cnt[BHRt + row] + p.cnt[2 * BHRt + row]);
        long long incl = n;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const long long v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        if (a < Rt) {
            off[a] = base + incl - n;
            if (a >= p.R) {
                p.cnt[row] = 0;
                p.cnt[BHRt + row] = 0;
                p.cnt[2 * BHRt + row] = Rt;
            }
        }
        base += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
        off[Rt] = base;
        if (base != (long long)(bh + 1) * per_head) atomicOr(p.status, DA2_DEV_BADINDEX);
    }
}

// One warp per (head, query region): the row's 16-bit key blocks ascending,
// then its 8-bit ones, then its 4-bit ones, at the row's offset.
__global__ void __launch_bounds__(128) lists_kernel(PlanArgs p) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const size_t row = (size_t)blockIdx.x * 4 + warp;
    const int R = p.R, Rt = p.Rt;
    if (row >= (size_t)p.BH * Rt) return;
    const int bh = (int)(row / Rt), a = (int)(row % Rt);
    uint16_t* krow = p.kidx + p.off[(size_t)bh * (Rt + 1) + a];
    if (a >= R) {
        // prefix row: every block, ascending (non-sparse, App. C.1)
        for (int b = lane; b < Rt; b += 32) krow[b] = (uint16_t)b;
        return;
    }
    const uint8_t* prow = p.prec + ((size_t)bh * R + a) * R;
    const unsigned lt = (1u << lane) - 1u;
    const size_t BHRt = (size_t)p.BH * Rt;
    // 16-bit: the video blocks of the budget, then every prefix block
    const int n16 = p.cnt[2 * BHRt + row] - p.Rp, n8 = p.cnt[row];
    for (int i = lane; i < p.Rp; i += 32) krow[n16 + i] = (uint16_t)(R + i);
    int i16 = 0, i8 = 0, i4 = 0;
    for (int b0 = 0; b0 < R; b0 += 32) {
        const int b = b0 + lane;
        const int pr = b < R ? prow[b] : 0;
        const unsigned m16 = __ballot_sync(0xffffffffu, pr == 16);
        const unsigned m8 = __ballot_sync(0xffffffffu, pr == 8);
        const unsigned m4 = __ballot_sync(0xffffffffu, pr == 4);
        if (pr == 16) krow[i16 + __popc(m16 & lt)] = (uint16_t)b;
        if (pr == 8) krow[n16 + p.Rp + i8 + __popc(m8 & lt)] = (uint16_t)b;
        if (pr == 4) krow[n16 + p.Rp + n8 + i4 + __popc(m4 & lt)] = (uint16_t)b;
        i16 += __popc(m16);
        i8 += __popc(m8);
        i4 += __popc(m4);
    }
}

// ---------------------------------------------------------------- per-row ranking
// Ranking option per query block (a reading of a per-query-row ranking; the
// pages rank all R^2 pairs of a head).  One CTA per row finds the C16-th,
// C8-th and Ck-th largest 76-bit keys K = (A bits : 0xFFF - b) -- A
// descending, ties to the smaller key block b (A >= 0, so its bits order as
// the values) -- by a radix selection over 8-bit digits in shared memory,
// then gives each key block 16 (K >= K_C16), 8 (K >= K_C8), 4 (K >= K_Ck) or
// 0 and counts the row's blocks per precision as the classification does.
constexpr int kRowRankThreads = 256;
typedef unsigned __int128 u128;

__global__ void __launch_bounds__(kRowRankThreads) row_rank_kernel(PlanArgs p, long long C16, long long C8,
                                                                   long long Ck) {
    constexpr int NT = kTargets;
    __shared__ unsigned hist[NT][256];
    __shared__ u128 pre[NT];        // selected prefix (digits in place)
    __shared__ int nbits[NT];       // bits of the prefix already fixed
    __shared__ long long need[NT];  // rank still sought inside the prefix (1-based)
    __shared__ uint8_t prec_s[4096];
    const int R = p.R, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const size_t row = blockIdx.x;
    const double* Arow = p.A + row * R;
    auto keyof = [&](int b) -> u128 {
        return ((u128)(unsigned long long)__double_as_longlong(Arow[b]) << 12) | (u128)(0xFFFu - (unsigned)b);
    };
    if (tid < NT) {
        pre[tid] = 0;
        nbits[tid] = 0;
        need[tid] = tid == 0 ? C16 : (tid == 1 ? C8 : Ck);
    }
    __syncthreads();
    for (int pass = 0; pass < 10; ++pass) {  // 76 bits in 8-bit digits (the last one 4 bits)
        for (int i = tid; i < NT * 256; i += kRowRankThreads) (&hist[0][0])[i] = 0u;
        __syncthreads();
        int w[NT], pos[NT];
        bool live[NT], any_live = false;
        for (int t = 0; t < NT; ++t) {
            live[t] = need[t] > 0 && nbits[t] < 76;
            w[t] = min(8, 76 - nbits[t]);
            pos[t] = 76 - nbits[t] - w[t];
            any_live = any_live || live[t];
        }
        if (!any_live) break;  // uniform: read from shared state after the barrier
        for (int b = tid; b < R; b += kRowRankThreads) {
            const u128 K = keyof(b);
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                if (!live[t]) continue;
                const int sh = 76 - nbits[t];
                if (sh < 128 && (K >> sh) != (pre[t] >> sh)) continue;
                atomicAdd(&hist[t][(unsigned)(K >> pos[t]) & ((1u << w[t]) - 1u)], 1u);
            }
        }
        __syncthreads();
        if (warp < NT && live[warp]) {
            const int t = warp;
            // lane covers bins [255 - 8 lane - 7, 255 - 8 lane], descending
            const int top = 255 - 8 * lane;
            unsigned sum = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) sum += hist[t][top - i];
            unsigned incl = sum;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const unsigned v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            const unsigned excl = incl - sum;
            const long long nd = need[t];
            if ((long long)excl < nd && nd <= (long long)incl) {
                long long cum = excl;
                for (int i = 0; i < 8; ++i) {
                    const int bin = top - i;
                    const long long c = hist[t][bin];
                    if (cum + c >= nd) {
                        need[t] = nd - cum;
                        pre[t] |= (u128)bin << pos[t];
                        nbits[t] += w[t];
                        break;
                    }
                    cum += c;
                }
            }
        }
        __syncthreads();
    }
    const u128 k16 = pre[0], k8 = pre[1], kk = pre[2];
    const bool has16 = C16 > 0, has8 = C8 > 0, hask = Ck > 0;
    for (int b = tid; b < R; b += kRowRankThreads) {
        const u128 K = keyof(b);
        prec_s[b] = (has16 && K >= k16) ? 16 : (has8 && K >= k8) ? 8 : ((hask && K >= kk) ? 4 : 0);
    }
    __syncthreads();
    uint8_t* prow = p.prec + row * R;
    for (int b = tid; b < R; b += kRowRankThreads) prow[b] = prec_s[b];
    if (tid < 32) {
        int n16 = 0, n8 = 0, n4 = 0;
        for (int b0 = 0; b0 < R; b0 += 32) {
            const int b = b0 + lane;
            const int pr = b < R ? prec_s[b] : 0;
            n16 += __popc(__ballot_sync(0xffffffffu, pr == 16));
            n8 += __popc(__ballot_sync(0xffffffffu, pr == 8));
            n4 += __popc(__ballot_sync(0xffffffffu, pr == 4));
        }
        if (lane == 0) {
            const size_t BHRt = (size_t)p.BH * p.Rt, rt = (row / R) * p.Rt + row % R;
            p.cnt[rt] = n8;
            p.cnt[BHRt + rt] = n4;
            p.cnt[2 * BHRt + rt] = n16 + p.Rp;  // every prefix key is kept at 16 bits
        }
    }
}

constexpr int kSelectPasses = 8;  // 12-bit digits cover the 96-bit key

}  // namespace

size_t plan_scratch_bytes(int BH, int R, int d) {
    size_t b = (size_t)BH * R * R * sizeof(double);        // max-branch logits
    b += (size_t)2 * BH * sizeof(unsigned long long);      // A bit range per head
    b = (b + 255) & ~(size_t)255;
    b += (size_t)kTargets * BH * sizeof(SelectTarget);
    b = (b + 255) & ~(size_t)255;
    b += (size_t)kTargets * BH * 4096 * sizeof(unsigned);
    b = (b + 255) & ~(size_t)255;
    b += (size_t)BH * sizeof(unsigned);
    b = (b + 255) & ~(size_t)255;
    b += (size_t)2 * BH * sizeof(int);  // candidate list counts and states
    b = (b + 255) & ~(size_t)255;
    b += mx_scratch_bytes(BH, R, d);  // split descriptors of the exact max-pool branch
    return b;
}

void plan_carve_scratch(PlanArgs* p, void* scratch) {
    char* c = static_cast<char*>(scratch);
    p->Lmax = reinterpret_cast<double*>(c);
    size_t off = (size_t)p->BH * p->R * p->R * sizeof(double);
    p->abits_minmax = reinterpret_cast<unsigned long long*>(c + off);
    off += (size_t)2 * p->BH * sizeof(unsigned long long);
    off = (off + 255) & ~(size_t)255;
    p->sel = reinterpret_cast<SelectTarget*>(c + off);
    off += (size_t)kTargets * p->BH * sizeof(SelectTarget);
    off = (off + 255) & ~(size_t)255;
    p->hist = reinterpret_cast<unsigned*>(c + off);
    off += (size_t)kTargets * p->BH * 4096 * sizeof(unsigned);
    off = (off + 255) & ~(size_t)255;
    p->done_count = reinterpret_cast<unsigned*>(c + off);
    off += (size_t)p->BH * sizeof(unsigned);
    off = (off + 255) & ~(size_t)255;
    p->cand_n = reinterpret_cast<int*>(c + off);
    off += (size_t)p->BH * sizeof(int);
    p->cand_state = reinterpret_cast<int*>(c + off);
    off += (size_t)p->BH * sizeof(int);
    off = (off + 255) & ~(size_t)255;
    mx_carve(p, c + off);
}

cudaError_t launch_plan(const PlanArgs& p, cudaStream_t stream) {
    const int R = p.R, BH = p.BH;
    const long long RR = (long long)R * R;
    // cumulative cuts of the ranking: 16-bit, 16+8-bit, kept
    const long long C16 = RR * p.bp16 / 10000, C8 = RR * (p.bp16 + p.bp8) / 10000,
                    Ck = RR * (p.bp16 + p.bp8 + p.bp4) / 10000;
    cudaError_t e;
    const double rd = 1.0 / sqrt((double)p.d);
    // the max-pool branch's logits of every block inside the exact range come
    // from integer tensor-core products; the fp64 chain below covers the rest
    if ((e = launch_max_logits(p, rd, stream)) != cudaSuccess) return e;
    dim3 lg((R + kLgTile - 1) / kLgTile, (R + kLgTile - 1) / kLgTile, 2 * BH);
    if (p.d == 64) {
        if ((e = cudaFuncSetAttribute(logits_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kLgSmem)) !=
            cudaSuccess)
            return e;
        logits_kernel<64><<<lg, kLgThreads, kLgSmem, stream>>>(p, rd);
    } else {
        if ((e = cudaFuncSetAttribute(logits_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kLgSmem)) !=
            cudaSuccess)
            return e;
        logits_kernel<128><<<lg, kLgThreads, kLgSmem, stream>>>(p, rd);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(p.abits_minmax, 0xFF, sizeof(unsigned long long) * BH, stream)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(p.abits_minmax + BH, 0, sizeof(unsigned long long) * BH, stream)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(p.hist, 0, sizeof(unsigned) * kTargets * 4096 * (size_t)BH, stream)) != cudaSuccess)
        return e;
    if ((e = cudaMemsetAsync(p.done_count, 0, sizeof(unsigned) * (size_t)BH, stream)) != cudaSuccess) return e;
    const size_t smem = sizeof(double) * 2 * R;
    if (smem > 48 * 1024) {
        e = cudaFuncSetAttribute(softmax_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    softmax_kernel<<<(unsigned)((size_t)BH * R), kSoftThreads, smem, stream>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // kept pairs of a head: the budgeted video pairs, plus every video row's
    // prefix keys and every prefix row's keys
    auto emit_lists = [&](long long budgeted) -> cudaError_t {
        const long long per_head = budgeted + (long long)R * p.Rp + (long long)p.Rp * p.Rt;
        offsets_kernel<<<(BH + 3) / 4, 128, 0, stream>>>(p, per_head);
        lists_kernel<<<(unsigned)(((size_t)BH * p.Rt + 3) / 4), 128, 0, stream>>>(p);
        return cudaGetLastError();
    };
    if (p.per_row) {
        // ranking per query block: quotas per row, no selection passes
        const long long C16r = (long long)R * p.bp16 / 10000, C8r = (long long)R * (p.bp16 + p.bp8) / 10000,
                        Ckr = (long long)R * (p.bp16 + p.bp8 + p.bp4) / 10000;
        row_rank_kernel<<<(unsigned)((size_t)BH * R), kRowRankThreads, 0, stream>>>(p, C16r, C8r, Ckr);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        return emit_lists((long long)R * Ckr);
    }
    select_init_kernel<<<(BH + 127) / 128, 128, 0, stream>>>(p, C16, C8, Ck);
    // about two 1024-thread CTAs per multiprocessor over all heads, so that
    // each CTA flushes its shared histogram once for many keys
    const long long per_head = std::max(1, 2 * std::max(1, p.num_sms) / BH);
    long long chunk = (RR + per_head - 1) / per_head;
    chunk = std::max<long long>(kHistMinChunk, (chunk + 4 * kHistThreads - 1) / (4 * kHistThreads) * (4 * kHistThreads));
    dim3 hg((unsigned)((RR + chunk - 1) / chunk), BH);
    // with no 16-bit tier its (empty) target is skipped: two live targets
    if (C16 > 0) {
        constexpr size_t hs = 3 * 4096 * sizeof(unsigned);
        if ((e = cudaFuncSetAttribute(select_hist_kernel<3>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)hs)) !=
            cudaSuccess)
            return e;
        for (int pass = 0; pass < kSelectPasses; ++pass)
            select_hist_kernel<3><<<hg, kHistThreads, hs, stream>>>(p, (int)chunk);
    } else {
        for (int pass = 0; pass < kSelectPasses; ++pass)
            select_hist_kernel<2><<<hg, kHistThreads, 2 * 4096 * sizeof(unsigned), stream>>>(p, (int)chunk);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    classify_kernel<<<(unsigned)(((size_t)BH * R + 3) / 4), 128, 0, stream>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    return emit_lists(Ck);
}

long long plan_kept_per_head(int Rv, int Rp, int bp16, int bp8, int bp4, int per_row) {
    const long long sum = bp16 + bp8 + bp4;
    const long long budgeted = per_row ? (long long)Rv * ((long long)Rv * sum / 10000) : (long long)Rv * Rv * sum / 10000;
    return budgeted + (long long)Rv * Rp + (long long)Rp * (Rv + Rp);
}

}  // namespace da2

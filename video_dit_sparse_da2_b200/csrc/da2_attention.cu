// da2_attention.cu -- phased block-sparse mixed-precision attention for
// sm_100a ("DraftAttention2", Sec. 3.3 "Phased execution" Eq. 7 and
// "Cross-precision accumulation" Eq. 8; App. B.3 shared normalization;
// App. C.1 formats and empty rows).
//
// Work item = two query blocks (a0, a1) of one head stacked into one M = 128
// tile: the block-scaled NVFP4 MMA has M = 128 per CTA, the method's query
// blocks have 64 tokens.  The pairs come from the handle's table (the same
// patch in two consecutive frames, whose lists are most alike in video).  The kernel walks the union of the
// two blocks' key lists phase by phase -- the 16-bit key blocks (when the
// plan has any), then the 8-bit ones, then the 4-bit ones, each ascending; a
// row takes part in a step only when its own block kept that key block at
// that precision, so every row sees exactly its own list in the order of the
// method.
//
// Roles (384 threads, two persistent CTAs per SM, each holding 256 of the 512
// tensor-memory columns; items fetched from a global counter):
//   warps 0-3  softmax: one thread per row of the tile (warp w reads
//              tensor-memory lanes 32w..32w+31, all 64 key columns of a step).
//              Reads S from tensor memory (then releases the S buffer at
//              once), keeps the row max m and the unquantized denominator l
//              (App. B.3), quantizes the weights into shared memory -- FP8:
//              e4m3 of p times the value tile scale over the phase unit, with
//              the fp32 rounding steps of the definition; NVFP4: per 16 keys a
//              ue4m3 scale from the group's largest weight (taken from the
//              group maximum of the scores) and e2m1 codes of p * (ratio *
//              1/scale), the definition's (p * ratio) * 1/scale reordered,
//              equal to it whenever p is a power of two; p of the winning key
//              is exactly 1 in both; 16-bit: bf16 of p.  Once the row max of
//              a step is known it posts the row's factor for O (running-max
//              correction times the change of units of Eq. 8 at a phase
//              switch) to the correction warp of its quarter.  At the end of
//              an item it hands each row's output scale (unit / l) to the
//              epilogue.
//   warps 4-7  correction and epilogue: one thread per row, same lane
//              quarters.  Per step they multiply the rows of O whose factor is
//              not 1 (after the previous PV has completed), off the softmax
//              warps' path; the step's PV waits for them and for the softmax
//              warps.  At the end of an item they multiply O by the output
//              scale, convert to bf16 and store each row at its original token
//              position, while the softmax warps already work on the next
//              item.
//   warp 8     MMA issue (whole warp, one elected lane issues): S = Q K^T
//              (tcgen05.mma kind::f8f6f4, kind::i8, kind::mxf4nvf4 block16 or
//              kind::f16) into the S buffer, O += P V into the single O
//              accumulator once the softmax warps published the step's P.
//   warp 9     loader (whole warp, one elected lane issues): bulk async copies
//              of the K / V tiles (pre-tiled by the preparation kernel) into a
//              3-stage ring, and the step record of each stage.
//   warps 10-11 scheduler: fetch the next work item and merge the two rows'
//              lists into the item's step list.
// Every mbarrier wait is bounded; a stuck wait sets the status word, all
// roles drain their own outstanding work and the CTA frees tensor memory
// before returning.
#include "da2_common.cuh"
#include "da2_kernels.h"

namespace da2 {

namespace {

constexpr int kStages = 3;
// Roles: softmax warps 0-3 (one thread per tile row, all 64 key columns of a
// step), correction and epilogue warps 4-7 (one thread per tile row), MMA
// warp 8, loader warp 9, scheduler warps 10-11 (the register budgets are set
// per warpgroup of four warps).
constexpr int kSoftmaxThreads = 128;
constexpr int kThreads = 384;
constexpr int kMmaWarp = 8, kLoadWarp = 9;
// Registers per thread: every thread starts with kRegLaunch (two CTAs of 384
// threads share the 64K registers of an SM); the warpgroups then move to
// their own budgets, whose sum is the CTA's allocation.
constexpr uint32_t kRegLaunch = 80, kRegSoftmax = 152, kRegCorr = 48, kRegAux = 40;
static_assert((kRegSoftmax + kRegCorr + kRegAux) * 128 == kRegLaunch * kThreads,
              "the warpgroup register budgets must add up to the launch allocation");
static_assert(2 * kRegLaunch * kThreads <= 65536, "two CTAs per SM");
constexpr int CW = 64;      // key columns per softmax thread
constexpr int NP = CW / 2;  // float2 pairs per softmax thread
constexpr uint32_t kTmemCols = 256;
// tensor-memory column map (per CTA)
constexpr uint32_t kColO = 0;      // O accumulator, D columns
constexpr uint32_t kColS = 128;    // S buffer, 64 columns
constexpr uint32_t kColSfq = 192;  // Q scale factors, 4 columns per 64-channel chunk
constexpr uint32_t kColSfk = 200;  // K scale factors, 4 columns
constexpr uint32_t kColSfp = 204;  // P scale factors, 2 buffers x 4 columns
constexpr uint32_t kColSfv = 212;  // V scale factors, 2 buffers x 4 columns
constexpr uint32_t kColMeta = 220; // step record (StepMeta) of the step whose S is in the S buffer

// Step of the merged list: key block (12 bits), phase (2: 0 = 8-bit, 1 = 4-bit,
// 2 = 16-bit), row mask (2).
__device__ __forceinline__ uint16_t make_entry(int kb, int phase, int mask) {
    return (uint16_t)(kb | (phase << 12) | (mask << 14));
}
__device__ __forceinline__ int entry_phase(uint32_t e) { return (e >> 12) & 3; }

__device__ __forceinline__ uint32_t kmajor_off(int row, int chunk, int row_bytes) {
    return ((row >> 3) * (row_bytes >> 4) + chunk) * 128 + (row & 7) * 16;
}

template <int D, bool T16>
struct Smem {
    // byte offsets inside the dynamic shared memory block
    static constexpr uint32_t q8 = 0;                          // 128 x D
    static constexpr uint32_t q4 = q8 + 128 * D;               // 128 x D/2
    static constexpr uint32_t sfq = q4 + 64 * D;               // D/64 atoms of 512
    static constexpr uint32_t q16 = sfq + 1024;                // 128 x 2D (16-bit path only)
    static constexpr uint32_t stage = q16 + (T16 ? 256 * D : 0);  // kStages x stage_bytes
    // K then V tiles of one step (bf16 tiles are twice the FP8 ones), then
    // the NVFP4 K and V scale-factor atoms
    static constexpr uint32_t kv_bytes = T16 ? 128 * D : 64 * D;
    static constexpr uint32_t k_off = 0, v_off = kv_bytes, ksf_off = 2 * kv_bytes, vsf_off = 2 * kv_bytes + 512;
    static constexpr uint32_t stage_bytes = 2 * kv_bytes + 1024;
    static constexpr uint32_t p = stage + kStages * stage_bytes;  // 2 P buffers: weights, then NVFP4 scales
    static constexpr uint32_t p_sf = T16 ? 128 * 128 : 128 * 64;  // bf16 weights are 128 bytes per row
    static constexpr uint32_t p_bytes = p_sf + 512;
    static constexpr uint32_t bitmap = p + 2 * p_bytes;        // 6 x 128 words
    static constexpr uint32_t rcp = bitmap + 6 * 128 * 4;      // 128 floats: 1/value of each ue4m3 code
    static constexpr uint32_t meta = rcp + 128 * 4;            // kStages x 32 copies of the StepMeta record
    static constexpr uint32_t list = meta + kStages * 512;     // 2R entries of 16 bits
};

// Per-step scalars shared by all rows: key-block size, score scale,
// value-scale ratio.  The loader writes 32 copies (one per tensor-memory lane
// of a quarter) into the stage's 512-byte record before it arms the stage
// barrier; the MMA thread copies the record into tensor memory next to S
// (tcgen05.cp, before the S MMA, so the S commit covers it) and the softmax
// threads load it together with S.
struct __align__(16) StepMeta {
    int nk;
    float ck;     // K tile scale (FP8) or NVFP4 tile scale
    float ratio;  // V tile scale over the phase unit
    int pad;
};

// x / 6 correctly rounded (q = x * RN(1/6), one fma residual correction).
__device__ __forceinline__ float div6(float x) {
    const float c = 0.16666667163372039794921875f;
    const float q = x * c;
    const float r = fmaf(-q, 6.0f, x);
    return fmaf(r, c, q);
}

// 64 consecutive fp32 columns of this warp's tensor-memory lanes into v[0..31]
// as pairs, and 4 columns of the step record into r: three loads (no single
// instruction wider than 32 registers) and one wait in one asm statement.
__device__ __forceinline__ void tmem_ld64x2_rec(uint32_t taddr, uint32_t raddr, float2 (&v)[32],
                                                uint32_t (&r)[4]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%68];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%70];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x4.b32 {%64,%65,%66,%67}, [%69];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=f"(v[0].x), "=f"(v[0].y), "=f"(v[1].x), "=f"(v[1].y), "=f"(v[2].x), "=f"(v[2].y), "=f"(v[3].x), "=f"(v[3].y), "=f"(v[4].x), "=f"(v[4].y), "=f"(v[5].x), "=f"(v[5].y), "=f"(v[6].x), "=f"(v[6].y), "=f"(v[7].x), "=f"(v[7].y), "=f"(v[8].x), "=f"(v[8].y), "=f"(v[9].x), "=f"(v[9].y), "=f"(v[10].x), "=f"(v[10].y), "=f"(v[11].x), "=f"(v[11].y), "=f"(v[12].x), "=f"(v[12].y), "=f"(v[13].x), "=f"(v[13].y), "=f"(v[14].x), "=f"(v[14].y), "=f"(v[15].x), "=f"(v[15].y), "=f"(v[16].x), "=f"(v[16].y), "=f"(v[17].x), "=f"(v[17].y), "=f"(v[18].x), "=f"(v[18].y), "=f"(v[19].x), "=f"(v[19].y), "=f"(v[20].x), "=f"(v[20].y), "=f"(v[21].x), "=f"(v[21].y), "=f"(v[22].x), "=f"(v[22].y), "=f"(v[23].x), "=f"(v[23].y), "=f"(v[24].x), "=f"(v[24].y), "=f"(v[25].x), "=f"(v[25].y), "=f"(v[26].x), "=f"(v[26].y), "=f"(v[27].x), "=f"(v[27].y), "=f"(v[28].x), "=f"(v[28].y), "=f"(v[29].x), "=f"(v[29].y), "=f"(v[30].x), "=f"(v[30].y), "=f"(v[31].x), "=f"(v[31].y),
          "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
        : "r"(taddr), "r"(raddr), "r"(taddr + 32)
        : "memory");
}

// Max of the 16 consecutive values v[b..b+7] (pairs).
template <int NP>
__device__ __forceinline__ float groupmax16_raw(const float2 (&v)[NP], int b) {
    const float t0 = max3f(v[b].x, v[b].y, v[b + 1].x), t1 = max3f(v[b + 1].y, v[b + 2].x, v[b + 2].y);
    const float t2 = max3f(v[b + 3].x, v[b + 3].y, v[b + 4].x), t3 = max3f(v[b + 4].y, v[b + 5].x, v[b + 5].y);
    const float t4 = max3f(v[b + 6].x, v[b + 6].y, v[b + 7].x);
    return max3f(max3f(t0, t1, t2), t3, fmaxf(t4, v[b + 7].y));
}


template <uint32_t N>
__device__ __forceinline__ void setmaxnreg_inc() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N>
__device__ __forceinline__ void setmaxnreg_dec() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
// CTA-wide named barrier 1 (barrier 0 is __syncthreads), reached from the
// ends of the role branches.
__device__ __forceinline__ void roles_done_barrier() { asm volatile("bar.sync 1, %0;" ::"n"(kThreads) : "memory"); }
// Named barrier 2 of the two scheduler warps.
__device__ __forceinline__ void sched_barrier() { asm volatile("bar.sync 2, 64;" ::: "memory"); }

// A work item published by the scheduler warps (item < 0: no more work).
struct ItemInfo {
    int item, n16e, n8e, n_ent;  // steps of the union list: n16e 16-bit, then n8e 8-bit, then 4-bit
};

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]),
        "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]),
        "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

template <int D, bool T16>
__global__ void __launch_bounds__(kThreads, T16 ? 1 : 2) attention_kernel(AttnArgs p) {
    using L = Smem<D, T16>;
    extern __shared__ __align__(1024) uint8_t smem[];
    // bar_empty[st] completes when the PV of a step in stage st has finished:
    // it frees the stage for the loader, frees that step's P buffer two steps
    // later, and tells the correction and epilogue warps that O holds the step.
    __shared__ uint64_t bar_q, bar_qfree, bar_sfq, bar_full[kStages], bar_empty[kStages], bar_s, bar_sfree, bar_p[2],
        bar_epi, bar_osc[2], bar_drain, bar_ready[2], bar_listfree, bar_infofree[2], bar_creq[4][2];
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_sh, item_sh;
    __shared__ int n_ent_sh[3];
    __shared__ ItemInfo info_sh[2];    // per item parity: the work item and its step counts
    __shared__ float oscale_sh[2][128];  // per item parity and row: unit / l, for the epilogue
    __shared__ float ofac_sh[2][128];    // per step parity and row: factor for O before the step's PV

    // warp index and everything derived from shared scalars are broadcast
    // from lane 0 so that the compiler treats them as warp-uniform
    const int tid = threadIdx.x, warp = warp_uniform(tid >> 5), lane = tid & 31;
    const int R = p.R, BH = p.B * p.H;
    const size_t BHR = (size_t)BH * R;
    const int pairs = p.npairs;
    const int items = BH * pairs;
    const int nwords = (R + 31) / 32;
    uint32_t* bitmap = reinterpret_cast<uint32_t*>(smem + L::bitmap);
    uint16_t* list = reinterpret_cast<uint16_t*>(smem + L::list);
    volatile int* abort_v = &abort_sh;

    if (tid == 0) {
        mbar_init(&bar_q, 1);
        mbar_init(&bar_qfree, 1);
        mbar_init(&bar_sfq, kSoftmaxThreads);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&bar_full[s], 1);
            mbar_init(&bar_empty[s], 1);
        }
        mbar_init(&bar_s, 1);
        mbar_init(&bar_sfree, 4);  // one arrive per softmax warp
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bar_p[s], 8);    // one arrive per softmax warp and per correction warp
            for (int q = 0; q < 4; ++q) mbar_init(&bar_creq[q][s], 1);  // a softmax warp's O factors
            mbar_init(&bar_osc[s], 4);  // the softmax warps wrote an item's output scales
            mbar_init(&bar_ready[s], 1);      // the scheduler published an item
            mbar_init(&bar_infofree[s], 4);   // the epilogue warps are done with an item
        }
        mbar_init(&bar_listfree, 6);  // loader, MMA warp and the four softmax warps read the list
        mbar_init(&bar_epi, 4);       // the epilogue warps read O of an item
        mbar_init(&bar_drain, 1);
        abort_sh = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&tmem_base_sh, kTmemCols);
        tmem_relinquish();
    }
    {
        float* rcp = reinterpret_cast<float*>(smem + L::rcp);
        for (int c = tid; c < 128; c += kThreads) rcp[c] = c ? __frcp_rn(e4m3_to_f32((uint8_t)c)) : 0.0f;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = warp_uniform(tmem_base_sh);

    uint32_t loads_issued = 0;  // loader: stage fills issued (for the final drain)
    bool mma_issued = false;

    // Every role runs its own loop over the items the scheduler publishes; the
    // warpgroups take their register budgets once, here: the epilogue and
    // issue warpgroups release registers, the softmax warpgroup takes them
    // (a request blocks until the CTA's pool can serve it, with no time limit,
    // so only the softmax warpgroup ever requests before the end).
    if (warp >= 8) {
        if constexpr (!T16) setmaxnreg_dec<kRegAux>();
        if (warp == kLoadWarp) {
            uint32_t gstep = 0;
            for (int k = 0;; ++k) {
                if (!__all_sync(0xffffffffu, mbar_wait(&bar_ready[k & 1], (k >> 1) & 1, abort_v, p.status, p.wait_ns)))
                    break;
                const int item = warp_uniform(info_sh[k & 1].item);
                if (item < 0) break;
                const int n16e = warp_uniform(info_sh[k & 1].n16e), n8e = warp_uniform(info_sh[k & 1].n8e),
                  n_ent = warp_uniform(info_sh[k & 1].n_ent);
                const int bh = item / pairs, pr = item % pairs;
                const int a0 = p.pairs[2 * pr], a1 = p.pairs[2 * pr + 1];
                const bool has1 = a1 >= 0;

                // ================================================== loader (whole warp, one elected lane issues)
                const size_t t0 = (size_t)bh * R + a0, t1 = (size_t)bh * R + (has1 ? a1 : a0);
                const uint32_t qb8 = 64 * D, qb4 = 32 * D;
                const float sig8 = __fdiv_rn(p.vmax[bh], 448.0f), sig4 = __fdiv_rn(p.vmax[BH + bh], 2688.0f);
                // Q of this item replaces Q of the previous one once the previous
                // item's MMAs (which read it) have completed
                if (k > 0 && !__all_sync(0xffffffffu, mbar_wait(&bar_qfree, (k - 1) & 1, abort_v, p.status, p.wait_ns)))
                    break;
                const uint32_t qb16 = T16 ? 128 * D : 0;
                mbar_expect_tx_w(&bar_q, (has1 ? 2u : 1u) * (qb8 + qb4 + qb16));
                // the 8-bit Q tile: INT8 codes when the 8-bit phase's QK^T is INT8
                const uint8_t* q8src = p.q8i ? reinterpret_cast<const uint8_t*>(p.q8i) : p.q8;
                bulk_g2s_w(smem + L::q8, q8src + t0 * qb8, qb8, &bar_q);
                bulk_g2s_w(smem + L::q4, p.q4 + t0 * qb4, qb4, &bar_q);
                if constexpr (T16) bulk_g2s_w(smem + L::q16, p.q16 + t0 * qb16, qb16, &bar_q);
                if (has1) {
                    bulk_g2s_w(smem + L::q8 + qb8, q8src + t1 * qb8, qb8, &bar_q);
                    bulk_g2s_w(smem + L::q4 + qb4, p.q4 + t1 * qb4, qb4, &bar_q);
                    if constexpr (T16) bulk_g2s_w(smem + L::q16 + qb16, p.q16 + t1 * qb16, qb16, &bar_q);
                }
                for (int j = 0; j < n_ent; ++j) {
                    const uint32_t g = gstep + j, st = g % kStages;
                    if (!__all_sync(0xffffffffu, mbar_wait(&bar_empty[st], ((g / kStages) & 1) ^ 1, abort_v, p.status,
                                                           p.wait_ns)))
                        break;
                    const uint32_t e = warp_uniform((uint32_t)list[j]);
                    const int kb = e & 0xFFF, ph = entry_phase(e);
                    const size_t tk = (size_t)bh * R + kb;
                    uint8_t* sb = smem + L::stage + st * L::stage_bytes;
                    {
                        // step record: lane i writes copy i (one 16-byte store per lane)
                        // (the 16-bit path has no tile scales and unit 1)
                        const int nk = p.n_a[kb];
                        const float ck = ph == 2   ? 1.0f
                                         : (ph == 0 && p.si8) ? p.si8[BHR + tk]
                                                              : p.scale[(ph ? 4 : 1) * BHR + tk];
                        const float vs = ph == 2 ? 1.0f : p.scale[(ph ? 5 : 2) * BHR + tk];
                        const float sg = ph == 2 ? 1.0f : (ph ? sig4 : sig8);
                        const float ratio = sg > 0.0f ? __fdiv_rn(vs, sg) : 0.0f;
                        reinterpret_cast<uint4*>(smem + L::meta + st * 512)[lane] =
                            make_uint4((uint32_t)nk, __float_as_uint(ck), __float_as_uint(ratio), 0u);
                        // visible to the tensor-core copy of the MMA warp, which
                        // waits on the arrive below
                        fence_proxy_async_smem();
                        __syncwarp();
                    }
                    if (T16 && ph == 2) {
                        mbar_expect_tx_w(&bar_full[st], 2 * 128 * D);
                        bulk_g2s_w(sb + L::k_off, p.k16 + tk * (128 * D), 128 * D, &bar_full[st]);
                        bulk_g2s_w(sb + L::v_off, p.v16 + tk * (128 * D), 128 * D, &bar_full[st]);
                    } else if (ph == 0) {
                        mbar_expect_tx_w(&bar_full[st], 2 * 64 * D);
                        const uint8_t* k8src = p.k8i ? reinterpret_cast<const uint8_t*>(p.k8i) : p.k8;
                        bulk_g2s_w(sb + L::k_off, k8src + tk * (64 * D), 64 * D, &bar_full[st]);
                        bulk_g2s_w(sb + L::v_off, p.v8 + tk * (64 * D), 64 * D, &bar_full[st]);
                    } else {
                        mbar_expect_tx_w(&bar_full[st], 2 * 32 * D + 1024);
                        bulk_g2s_w(sb + L::k_off, p.k4 + tk * (32 * D), 32 * D, &bar_full[st]);
                        bulk_g2s_w(sb + L::v_off, p.v4 + tk * (32 * D), 32 * D, &bar_full[st]);
                        bulk_g2s_w(sb + L::ksf_off, p.sfk + tk * 512, 512, &bar_full[st]);
                        bulk_g2s_w(sb + L::vsf_off, p.sfv + tk * 512, 512, &bar_full[st]);
                    }
                    ++loads_issued;
                }

                if (lane == 0) mbar_arrive(&bar_listfree);
                gstep += n_ent;
            }
        } else if (warp == kMmaWarp) {
            uint32_t gstep = 0;
            for (int k = 0;; ++k) {
                if (!__all_sync(0xffffffffu, mbar_wait(&bar_ready[k & 1], (k >> 1) & 1, abort_v, p.status, p.wait_ns)))
                    break;
                const int item = warp_uniform(info_sh[k & 1].item);
                if (item < 0) break;
                const int n16e = warp_uniform(info_sh[k & 1].n16e), n8e = warp_uniform(info_sh[k & 1].n8e),
                  n_ent = warp_uniform(info_sh[k & 1].n_ent);

                // ================================================== MMA issue (whole warp, one elected lane issues)
                auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
                    return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_v, p.status, p.wait_ns));
                };
                bool ok = wait_all(&bar_q, k & 1);
                ok = ok && wait_all(&bar_sfq, k & 1);
                tc_fence_after();
                if (ok && n_ent > n16e + n8e) {
                    for (int ch = 0; ch < D / 64; ++ch)
                        tc_cp_32x128_x4_w(tmem + kColSfq + 4 * ch, sdesc(smem + L::sfq + 512 * ch, 128, 128));
                }
                // Descriptors of the fixed buffers; a stage or P buffer is selected
                // by adding its byte offset / 16 to the start-address field (bits
                // 0-13, which hold the shared-memory address / 16 without carry
                // since shared memory ends below 256 KB).
                const uint64_t dq8 = sdesc(smem + L::q8, 128, 8 * D), dq4 = sdesc(smem + L::q4, 128, 4 * D);
                const uint64_t dst = sdesc(smem + L::stage, 0, 0);  // stage base: lbo / sbo added per operand
                auto with_lbo_sbo = [](uint64_t d, uint32_t off, uint32_t lbo, uint32_t sbo) -> uint64_t {
                    return d + (off >> 4) + ((uint64_t)(lbo >> 4) << 16) + ((uint64_t)(sbo >> 4) << 32);
                };
                const uint64_t dmeta = sdesc(smem + L::meta, 128, 128);
                const bool qk_i8 = p.q8i != nullptr;  // the 8-bit phase's QK^T in INT8 (s32 scores)
                const uint64_t dp8 = sdesc(smem + L::p, 128, 512), dp4 = sdesc(smem + L::p, 128, 256);
                const uint64_t dpsf = sdesc(smem + L::p + L::p_sf, 128, 128);
                auto issue_pv = [&](int i) -> bool {
                    const uint32_t g = gstep + i, pb = g & 1, st = g % kStages;
                    // P of step g is written (and O rescaled for it); the first PV of
                    // an item overwrites O, which the epilogue of the previous item
                    // must have read
                    if (!wait_all(&bar_p[pb], (g >> 1) & 1)) return false;
                    if (i == 0 && k > 0 && !wait_all(&bar_epi, (k - 1) & 1)) return false;
                    tc_fence_after();
                    const int ph = entry_phase(warp_uniform((uint32_t)list[i]));
                    const uint32_t so = st * L::stage_bytes;
                    const uint64_t po = (pb * L::p_bytes) >> 4;
                    if (T16 && ph == 2) {
                        // bf16 P (128-byte rows) x bf16 V^T, K = 16 keys per MMA
                        const uint64_t dp16 = sdesc(smem + L::p, 128, 1024);
                        const uint64_t dv16 = with_lbo_sbo(dst, so + L::v_off, 128, 1024);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma_bf16_w(tmem + kColO, dp16 + po + 16 * kk, dv16 + 16 * kk, idesc_bf16(128, D),
                                       (i > 0 || kk > 0) ? 1u : 0u);
                    } else if (ph == 0) {
                        const uint64_t dv8 = with_lbo_sbo(dst, so + L::v_off, 128, 512);
#pragma unroll
                        for (int kk = 0; kk < 2; ++kk)
                            mma_f8_w(tmem + kColO, dp8 + po + 16 * kk, dv8 + 16 * kk, idesc_f8(128, D),
                                     (i > 0 || kk > 0) ? 1u : 0u);
                    } else {
                        tc_cp_32x128_x4_w(tmem + kColSfp + 4 * pb, dpsf + po);
                        tc_cp_32x128_x4_w(tmem + kColSfv + 4 * pb, with_lbo_sbo(dst, so + L::vsf_off, 128, 128));
                        mma_f4_w(tmem + kColO, dp4 + po, with_lbo_sbo(dst, so + L::v_off, 128, 256), idesc_f4(128, D),
                                 tmem + kColSfp + 4 * pb, tmem + kColSfv + 4 * pb, i > 0 ? 1u : 0u);
                    }
                    // frees the stage and (two steps later) the P buffer, and tells
                    // the correction and epilogue warps that O holds step g
                    tc_commit_w(&bar_empty[st]);
                    return true;
                };
                for (int j = 0; j < n_ent && ok; ++j) {
                    const uint32_t g = gstep + j, st = g % kStages;
                    if (!wait_all(&bar_full[st], (g / kStages) & 1)) {
                        ok = false;
                        break;
                    }
                    // the S buffer is free once every softmax warp has read step g-1
                    if (g > 0 && !wait_all(&bar_sfree, (g - 1) & 1)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int ph = entry_phase(warp_uniform((uint32_t)list[j]));
                    const uint32_t so = st * L::stage_bytes;
                    const uint32_t sd = tmem + kColS;
                    // step record next to S (the previous one was read with S(g-1))
                    tc_cp_32x128_x4_w(tmem + kColMeta, dmeta + st * (512 >> 4));
                    if (T16 && ph == 2) {
                        // bf16 Q (2D-byte rows) x bf16 K, K = 16 channels per MMA
                        const uint64_t dq16 = sdesc(smem + L::q16, 128, 16 * D);
                        const uint64_t dk16 = with_lbo_sbo(dst, so + L::k_off, 128, 16 * D);
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk)
                            mma_bf16_w(sd, dq16 + 16 * kk, dk16 + 16 * kk, idesc_bf16(128, 64), kk > 0 ? 1u : 0u);
                    } else if (ph == 0) {
                        const uint64_t dk8 = with_lbo_sbo(dst, so + L::k_off, 128, 8 * D);
#pragma unroll
                        for (int kk = 0; kk < D / 32; ++kk) {
                            if (qk_i8)
                                mma_i8_w(sd, dq8 + 16 * kk, dk8 + 16 * kk, idesc_i8(128, 64), kk > 0 ? 1u : 0u);
                            else
                                mma_f8_w(sd, dq8 + 16 * kk, dk8 + 16 * kk, idesc_f8(128, 64), kk > 0 ? 1u : 0u);
                        }
                    } else {
                        tc_cp_32x128_x4_w(tmem + kColSfk, with_lbo_sbo(dst, so + L::ksf_off, 128, 128));
                        const uint64_t dk4 = with_lbo_sbo(dst, so + L::k_off, 128, 4 * D);
#pragma unroll
                        for (int kk = 0; kk < D / 64; ++kk)
                            mma_f4_w(sd, dq4 + 16 * kk, dk4 + 16 * kk, idesc_f4(128, 64), tmem + kColSfq + 4 * kk,
                                     tmem + kColSfk + 2 * kk, kk > 0 ? 1u : 0u);
                    }
                    tc_commit_w(&bar_s);
                    mma_issued = true;
                    if (j > 0 && !issue_pv(j - 1)) {
                        ok = false;
                        break;
                    }
                }
                if (ok && n_ent > 0) ok = issue_pv(n_ent - 1);

                // Q of this item is free once its MMAs have completed
                tc_commit_w(&bar_qfree);
                if (lane == 0) mbar_arrive(&bar_listfree);
                gstep += n_ent;
            }
        } else {
            // ================================================== scheduler (warps 10-11)
            // fetches work items and builds each item's merged step list: the
            // union of the two rows' lists per phase
            const int stid = tid - 10 * 32;
            for (int k = 0;; ++k) {
                // the list of item k-1 has been read, and the epilogue warps
                // are done with the item record of item k-2
                bool ok = true;
                if (k > 0) ok = mbar_wait(&bar_listfree, (k - 1) & 1, abort_v, p.status, p.wait_ns);
                if (ok && k > 1) ok = mbar_wait(&bar_infofree[k & 1], ((k - 2) >> 1) & 1, abort_v, p.status, p.wait_ns);
                if (stid == 0) item_sh = atomicAdd(p.work_counter, 1);
                sched_barrier();
                const int item = item_sh;
                const bool stop = item >= items || *abort_v || !ok;
                sched_barrier();
                if (stop) {
                    if (stid == 0) {
                        info_sh[k & 1].item = -1;
                        mbar_arrive(&bar_ready[k & 1]);
                    }
                    break;
                }
                const int bh = item / pairs, pr = item % pairs;
                const int a0 = p.pairs[2 * pr], a1 = p.pairs[2 * pr + 1];
                const bool has1 = a1 >= 0;
                constexpr int nph = T16 ? 3 : 2;  // phases 0 (8-bit), 1 (4-bit), 2 (16-bit)
                for (int i = stid; i < 2 * nph * nwords; i += 64) bitmap[i] = 0u;
                sched_barrier();
                for (int hf = 0; hf < (has1 ? 2 : 1); ++hf) {
                    const size_t row = (size_t)bh * R + (hf ? a1 : a0);
                    const int n8 = p.cnt[row], n4 = p.cnt[BHR + row], n16 = p.cnt[2 * BHR + row];
                    // without the bf16 operands there is no 16-bit phase: a plan
                    // with 16-bit pairs is an error here (reported and skipped)
                    if (!T16 && n16 > 0 && stid == 0) atomicOr(p.status, DA2_DEV_BADINDEX);
                    const uint16_t* L0 = p.kidx + p.off[(size_t)bh * (R + 1) + (hf ? a1 : a0)];
                    for (int i = (T16 ? 0 : n16) + stid; i < n16 + n8 + n4; i += 64) {
                        const int kb = L0[i];
                        if (kb >= R) {
                            atomicOr(p.status, DA2_DEV_BADINDEX);
                            continue;
                        }
                        const int ph = i < n16 ? 2 : (i < n16 + n8 ? 0 : 1);
                        atomicOr(&bitmap[(ph * 2 + hf) * nwords + (kb >> 5)], 1u << (kb & 31));
                    }
                }
                sched_barrier();
                if (warp == 10) {
                    int base = 0;
                    // union list in phase order: 16-bit, 8-bit, 4-bit
                    for (int oi = 0; oi < nph; ++oi) {
                        const int ph = T16 ? (oi == 0 ? 2 : oi - 1) : oi;
                        const int before = base;
                        for (int w0 = 0; w0 < nwords; w0 += 32) {
                            const int w = w0 + lane;
                            const uint32_t m0 = w < nwords ? bitmap[(ph * 2 + 0) * nwords + w] : 0u;
                            const uint32_t m1 = w < nwords ? bitmap[(ph * 2 + 1) * nwords + w] : 0u;
                            uint32_t u = m0 | m1;
                            const int c = __popc(u);
                            int incl = c;
#pragma unroll
                            for (int o = 1; o < 32; o <<= 1) {
                                const int v = __shfl_up_sync(0xffffffffu, incl, o);
                                if (lane >= o) incl += v;
                            }
                            int pos = base + incl - c;
                            while (u) {
                                const int bit = __ffs(u) - 1;
                                u &= u - 1;
                                const int mask = ((m0 >> bit) & 1) | (((m1 >> bit) & 1) << 1);
                                list[pos++] = make_entry(w * 32 + bit, ph, mask);
                            }
                            base += __shfl_sync(0xffffffffu, incl, 31);
                        }
                        if (lane == 0) n_ent_sh[ph] = base - before;
                        __syncwarp();
                    }
                    if (lane == 0) {
                        info_sh[k & 1].item = item;
                        info_sh[k & 1].n16e = T16 ? n_ent_sh[2] : 0;
                        info_sh[k & 1].n8e = n_ent_sh[0];
                        info_sh[k & 1].n_ent = base;
                        // the arrive publishes the list and the record (release)
                        mbar_arrive(&bar_ready[k & 1]);
                    }
                }
            }
        }
        roles_done_barrier();
        if constexpr (!T16) setmaxnreg_inc<kRegLaunch>();
    } else if (warp < 4) {
        if constexpr (!T16) setmaxnreg_inc<kRegSoftmax>();
        uint32_t gstep = 0;
        for (int k = 0;; ++k) {
                if (!__all_sync(0xffffffffu, mbar_wait(&bar_ready[k & 1], (k >> 1) & 1, abort_v, p.status, p.wait_ns)))
                    break;
                const int item = warp_uniform(info_sh[k & 1].item);
                if (item < 0) break;
                const int n16e = warp_uniform(info_sh[k & 1].n16e), n8e = warp_uniform(info_sh[k & 1].n8e),
                      n_ent = warp_uniform(info_sh[k & 1].n_ent);
                const int bh = item / pairs, pr = item % pairs;
                const int a0 = p.pairs[2 * pr], a1 = p.pairs[2 * pr + 1];
                const bool has1 = a1 >= 0;

                // ================================================== softmax
                const int quarter = warp;                       // tensor-memory lane quarter
                const int r = 32 * quarter + lane;              // tile row
                const int hf = quarter >> 1;                    // which query block of the pair (= r >> 6)
                const bool qvalid = hf == 0 || has1;
                const int a = qvalid && hf ? a1 : a0;
                const size_t ta = (size_t)bh * R + (qvalid ? a : a0);
                const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
                const float rdl2e = (D == 64 ? 0.125f : 0.0883883461356163025f) * 1.4426950408889634f;
                const float* rcp_tab = reinterpret_cast<const float*>(smem + L::rcp);
                // Q scale factors of this row into the copy atoms (one per 64 channels)
                for (int ch = 0; ch < D / 64; ++ch) {
                    uint8_t* atom = smem + L::sfq;
                    const uint8_t* src = p.sfq + ta * (64 * (D / 16)) + (r & 63) * (D / 16);
                    const uint32_t w = qvalid ? *reinterpret_cast<const uint32_t*>(src + 4 * ch) : 0u;
                    *reinterpret_cast<uint32_t*>(atom + 512 * ch + 16 * (r & 31) + 4 * (r >> 5)) = w;
                }
                fence_proxy_async_smem();
                mbar_arrive(&bar_sfq);
                const bool qk_i8 = p.q8i != nullptr;  // 8-bit phase scores are int32 from INT8 operands
                const float sq8 = qk_i8 ? p.si8[ta] : p.scale[ta], gq4 = p.scale[3 * BHR + ta];
                const float sig8 = __fdiv_rn(p.vmax[bh], 448.0f), sig4 = __fdiv_rn(p.vmax[BH + bh], 2688.0f);
                // changes of units between the phases (Eq. 8): O / u_old -> O / u_new,
                // with unit 1 for the 16-bit phase
                const float switch_f = sig4 > 0.0f ? __fdiv_rn(sig8, sig4) : 1.0f;
                const float f16_8 = sig8 > 0.0f ? __fdiv_rn(1.0f, sig8) : 1.0f;
                const float f16_4 = sig4 > 0.0f ? __fdiv_rn(1.0f, sig4) : 1.0f;
                // row factors of the score scale, in log2 units
                const float cq8 = sq8 * rdl2e, cq4 = gq4 * rdl2e;
                float m = -INFINITY, l = 0.0f;  // l: this thread's share of the denominator
                bool ok = true;
                uint32_t e_next = warp_uniform(n_ent > 0 ? (uint32_t)list[0] : 0u);
                for (int j = 0; j < n_ent && ok; ++j) {
                    const uint32_t g = gstep + j, pb = g & 1;
                    const uint32_t e = e_next;
                    if (j + 1 < n_ent) e_next = warp_uniform((uint32_t)list[j + 1]);
                    const int ph = entry_phase(e);
                    const bool active = (e >> (14 + hf)) & 1;
                    // S of step g and its step record
                    const bool waited = mbar_wait(&bar_s, g & 1, abort_v, p.status, p.wait_ns);
                    if (!__all_sync(0xffffffffu, waited)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    float2 v[NP];
                    StepMeta mt;
                    if (active) {
                        uint32_t mw[4];
                        tmem_ld64x2_rec(lane_base + kColS, lane_base + kColMeta, v, mw);
                        mt.nk = (int)mw[0];
                        mt.ck = __uint_as_float(mw[1]);
                        mt.ratio = __uint_as_float(mw[2]);
                    }
                    // the warp's loads of S are complete (their wait is warp-wide):
                    // one arrive per warp
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bar_sfree);
                    // P buffer pb was last read by the PV of step g-2, which the MMA
                    // warp issued before S(g): the S commit awaited above covers it
                    uint8_t* pbuf = smem + L::p + pb * L::p_bytes;
                    // Factor for O before this step's PV, handed to the correction
                    // warp of this lane quarter as soon as it is known: the
                    // running-max correction, times the change of units (Eq. 8) at
                    // a phase switch, which applies to every row.  The factor buffer
                    // of parity pb was read for step g-2 before that step's PV,
                    // which the MMA warp issued before S(g).
                    auto post_factor = [&](float c) {
                        float f = c;
                        if (j > 0 && j == n16e && n8e > 0) f *= f16_8;                   // 16-bit -> 8-bit units
                        if (j > 0 && j == n16e + n8e) f *= n8e > 0 ? switch_f : f16_4;  // -> 4-bit units
                        ofac_sh[pb][r] = j > 0 ? f : 1.0f;
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&bar_creq[quarter][pb]);
                    };
                    float corr = 1.0f;
                    if (active) {
                        // v = s * c (log2 units); the winning key gets v - m = 0
                        // exactly, hence p = 1 exactly, as in the definition: the
                        // product p * ratio then meets the same e4m3 / e2m1
                        // rounding ties as p = e^(s - m) computed exactly.
                        const float c2 = (ph == 2 ? rdl2e : (ph ? cq4 : cq8)) * mt.ck;
                        const float2 c22 = make_float2(c2, c2);
                        if (qk_i8 && ph == 0) {
                            // int32 scores (|S| < 127^2 * 128 < 2^22) to float, exactly:
                            // S + 1.5 * 2^23 as float bits, minus 1.5 * 2^23
                            const float2 magic = make_float2(-12582912.0f, -12582912.0f);
#pragma unroll
                            for (int i = 0; i < NP; ++i) {
                                const float2 b = make_float2(__int_as_float(__float_as_int(v[i].x) + 0x4B400000),
                                                             __int_as_float(__float_as_int(v[i].y) + 0x4B400000));
                                v[i] = __fadd2_rn(b, magic);
                            }
                        }
#pragma unroll
                        for (int i = 0; i < NP; ++i) v[i] = __fmul2_rn(v[i], c22);
                        const int nk = mt.nk;  // valid keys of the block
                        if (nk < CW) {
                            if (nk >= CW - 16) {
#pragma unroll
                                for (int i = NP - 8; i < NP; ++i) {
                                    if (2 * i >= nk) v[i].x = -INFINITY;
                                    if (2 * i + 1 >= nk) v[i].y = -INFINITY;
                                }
                            } else {
#pragma unroll
                                for (int i = 0; i < NP; ++i) {
                                    if (2 * i >= nk) v[i].x = -INFINITY;
                                    if (2 * i + 1 >= nk) v[i].y = -INFINITY;
                                }
                            }
                        }
                        // maxima of the 16-key groups (they also give the NVFP4
                        // group scales below) and of the row
                        constexpr int NGR = CW / 16;
                        float gm[NGR];
#pragma unroll
                        for (int gi = 0; gi < NGR; ++gi) gm[gi] = groupmax16_raw<NP>(v, 8 * gi);
                        float rmx = gm[0];
#pragma unroll
                        for (int gi = 1; gi < NGR; gi += 2)
                            rmx = gi + 1 < NGR ? max3f(rmx, gm[gi], gm[gi + 1]) : fmaxf(rmx, gm[gi]);
                        const float mn = fmaxf(m, rmx);
                        if (m != -INFINITY && mn > m) corr = ex2f(m - mn);
                        m = mn;
                        post_factor(corr);
                        const float2 nm = make_float2(-mn, -mn);
                        const float2 rt = make_float2(mt.ratio, mt.ratio);
                        float2 acc0 = make_float2(0.0f, 0.0f), acc1 = acc0;
                        // p = 2^(v - m) and x = p * ratio for the 16 keys of a group (b = first pair)
                        auto exp_group = [&](int b) {
#pragma unroll
                            for (int i = b; i < b + 8; i += 2) {
                                const float2 t0 = __fadd2_rn(v[i], nm), t1 = __fadd2_rn(v[i + 1], nm);
                                const float2 p0 = make_float2(ex2f(t0.x), ex2f(t0.y));
                                const float2 p1 = make_float2(ex2f(t1.x), ex2f(t1.y));
                                acc0 = __fadd2_rn(acc0, p0);
                                acc1 = __fadd2_rn(acc1, p1);
                                v[i] = __fmul2_rn(p0, rt);
                                v[i + 1] = __fmul2_rn(p1, rt);
                            }
                        };
                        // Each phase computes and quantizes group by group inside its
                        // own branch, so the exponentials of one group overlap the
                        // conversions of the previous one.
                        if (T16 && ph == 2) {
                            // 16-bit path: weights bf16(p) (round to nearest even), unit 1
#pragma unroll
                            for (int ch = 0; ch < CW / 16; ++ch) {
                                const int b = ch * 8;
                                exp_group(b);
                                uint32_t w[8];
#pragma unroll
                                for (int i = 0; i < 8; ++i) {
                                    const __nv_bfloat162 b2 = __floats2bfloat162_rn(v[b + i].x, v[b + i].y);
                                    w[i] = *reinterpret_cast<const uint32_t*>(&b2);
                                }
                                *reinterpret_cast<uint4*>(pbuf + kmajor_off(r, 2 * ch, 128)) =
                                    make_uint4(w[0], w[1], w[2], w[3]);
                                *reinterpret_cast<uint4*>(pbuf + kmajor_off(r, 2 * ch + 1, 128)) =
                                    make_uint4(w[4], w[5], w[6], w[7]);
                            }
                        } else if (ph == 0) {
#pragma unroll
                            for (int ch = 0; ch < CW / 16; ++ch) {
                                const int b = ch * 8;
                                exp_group(b);
                                *reinterpret_cast<uint4*>(pbuf + kmajor_off(r, ch, 64)) =
                                    make_uint4(pack_e4m3x4(v[b], v[b + 1]), pack_e4m3x4(v[b + 2], v[b + 3]),
                                               pack_e4m3x4(v[b + 4], v[b + 5]), pack_e4m3x4(v[b + 6], v[b + 7]));
                            }
                        } else {
                            // Group scale from the group maximum: p is monotonic in v
                            // and rounding is monotonic, so the largest weight of the
                            // group is 2^(max v - m) * ratio rounded as each weight
                            // is.  Scale code and 1/value are known before the weights.
                            uint32_t sfw = 0, wq[CW / 8];
                            float rcs[NGR];
#pragma unroll
                            for (int gi = 0; gi < NGR; ++gi) {
                                const float ym = ex2f(gm[gi] - m) * mt.ratio;
                                const uint32_t sf = cvt_e4m3x2(div6(ym), 0.0f);
                                rcs[gi] = rcp_tab[sf];  // 0 for code 0: every weight of the group 0
                                sfw |= sf << (8 * gi);
                            }
                            // weights p * (ratio * 1/value): the same value as
                            // (p * ratio) * 1/value when p is a power of two, in
                            // particular p = 1 for the row maximum
#pragma unroll
                            for (int gi = 0; gi < NGR; ++gi) {
                                const float sgv = mt.ratio * rcs[gi];
                                const float2 sg2 = make_float2(sgv, sgv);
                                float2 y[8];
#pragma unroll
                                for (int i = 0; i < 8; ++i) {
                                    const float2 tt = __fadd2_rn(v[8 * gi + i], nm);
                                    const float2 pp = make_float2(ex2f(tt.x), ex2f(tt.y));
                                    if (i & 1) acc1 = __fadd2_rn(acc1, pp);
                                    else acc0 = __fadd2_rn(acc0, pp);
                                    y[i] = __fmul2_rn(pp, sg2);
                                }
                                wq[2 * gi] = pack_e2m1x8(y[0], y[1], y[2], y[3]);
                                wq[2 * gi + 1] = pack_e2m1x8(y[4], y[5], y[6], y[7]);
                            }
                            // 32 keys = one 16-byte chunk of the 32-byte row
#pragma unroll
                            for (int ch = 0; ch < CW / 32; ++ch)
                                *reinterpret_cast<uint4*>(pbuf + kmajor_off(r, ch, 32)) =
                                    make_uint4(wq[4 * ch], wq[4 * ch + 1], wq[4 * ch + 2], wq[4 * ch + 3]);
                            uint8_t* sfp = pbuf + L::p_sf + 16 * (r & 31) + 4 * (r >> 5);
                            *reinterpret_cast<uint32_t*>(sfp) = sfw;
                        }
                        const float2 a2 = __fadd2_rn(acc0, acc1);
                        l = l * corr + (a2.x + a2.y);
                    } else {
                        // row not in this step: zero weights
                        post_factor(1.0f);
                        if (T16 && ph == 2) {
#pragma unroll
                            for (int ch = 0; ch < 8; ++ch)
                                *reinterpret_cast<uint4*>(pbuf + kmajor_off(r, ch, 128)) = make_uint4(0, 0, 0, 0);
                        } else if (ph == 0) {
#pragma unroll
                            for (int ch = 0; ch < CW / 16; ++ch)
                                *reinterpret_cast<uint4*>(pbuf + kmajor_off(r, ch, 64)) =
                                    make_uint4(0, 0, 0, 0);
                        } else {
#pragma unroll
                            for (int ch = 0; ch < CW / 32; ++ch)
                                *reinterpret_cast<uint4*>(pbuf + kmajor_off(r, ch, 32)) =
                                    make_uint4(0, 0, 0, 0);
                            uint8_t* sfp = pbuf + L::p_sf + 16 * (r & 31) + 4 * (r >> 5);
                            *reinterpret_cast<uint32_t*>(sfp) = 0u;
                        }
                    }
                    // every thread makes its weight stores visible to the tensor
                    // core; after the warp barrier one lane publishes them
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bar_p[pb]);
                }
                // output scale of each row for the epilogue warps (unit of the last
                // phase over the unquantized denominator; 0 for a row with no key)
                {
                    const float unit = n_ent > n16e + n8e ? sig4 : (n8e > 0 ? sig8 : 1.0f);
                    oscale_sh[k & 1][r] = (ok && l > 0.0f) ? __fdiv_rn(unit, l) : 0.0f;
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bar_osc[k & 1]);
                }

            if (lane == 0) mbar_arrive(&bar_listfree);
            gstep += n_ent;
        }
        if constexpr (!T16) setmaxnreg_dec<kRegLaunch>();
        roles_done_barrier();
    } else {
        if constexpr (!T16) setmaxnreg_dec<kRegCorr>();
        uint32_t gstep = 0;
        for (int k = 0;; ++k) {
                if (!__all_sync(0xffffffffu, mbar_wait(&bar_ready[k & 1], (k >> 1) & 1, abort_v, p.status, p.wait_ns)))
                    break;
                const int item = warp_uniform(info_sh[k & 1].item);
                if (item < 0) break;
                const int n16e = warp_uniform(info_sh[k & 1].n16e), n8e = warp_uniform(info_sh[k & 1].n8e),
                      n_ent = warp_uniform(info_sh[k & 1].n_ent);
                const int bh = item / pairs, pr = item % pairs;
                const int a0 = p.pairs[2 * pr], a1 = p.pairs[2 * pr + 1];
                const bool has1 = a1 >= 0;

                // ================================================== epilogue
                const int quarter = warp - 4;
                const int r = 32 * quarter + lane;
                const int hf = quarter >> 1;
                const bool qvalid = hf == 0 || has1;
                const int a = qvalid && hf ? a1 : a0;
                const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
                // ---- O correction, step by step: once the softmax warp of this
                // quarter posted the step's factors, rows whose factor is not 1
                // are rescaled in O (which must hold the PV of the previous step
                // first), then this warp's arrive completes, with the softmax
                // warps', the step's P barrier
                bool cok = true;
                for (int j = 0; j < n_ent; ++j) {
                    const uint32_t g = gstep + j, pb = g & 1;
                    if (!__all_sync(0xffffffffu,
                                    mbar_wait(&bar_creq[quarter][pb], (g >> 1) & 1, abort_v, p.status, p.wait_ns))) {
                        cok = false;
                        break;
                    }
                    const float f = ofac_sh[pb][r];
                    if (__any_sync(0xffffffffu, f != 1.0f)) {
                        // a factor other than 1 only from the second step on
                        const uint32_t gp = g - 1;
                        const bool w2 =
                            mbar_wait(&bar_empty[gp % kStages], (gp / kStages) & 1, abort_v, p.status, p.wait_ns);
                        if (!__all_sync(0xffffffffu, w2)) {
                            cok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint64_t f2 = pack2(f, f);
#pragma unroll 1
                        for (int c0 = 0; c0 < D; c0 += 32) {
                            uint32_t o[32];
                            tmem_ld32(lane_base + kColO + c0, o);
#pragma unroll
                            for (int c = 0; c < 32; c += 2) {
                                const uint64_t x = mul2(pack2(__uint_as_float(o[c]), __uint_as_float(o[c + 1])), f2);
                                o[c] = __float_as_uint(lo2(x));
                                o[c + 1] = __float_as_uint(hi2(x));
                            }
                            tmem_st32(lane_base + kColO + c0, o);
                        }
                        tc_wait_st();
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bar_p[pb]);
                }
                // ---- epilogue: the softmax warps' output scales of this item
                bool ok = cok && __all_sync(0xffffffffu, mbar_wait(&bar_osc[k & 1], (k >> 1) & 1, abort_v, p.status, p.wait_ns));
                float o_scale = 0.0f;
                const bool have = n_ent > 0 && ok;
                if (have) {
                    // O holds the item once its last PV has completed
                    const uint32_t g = gstep + n_ent - 1;
                    if (!mbar_wait(&bar_empty[g % kStages], (g / kStages) & 1, abort_v, p.status, p.wait_ns)) ok = false;
                    tc_fence_after();
                    o_scale = oscale_sh[k & 1][r];
                }
                const bool have_o = __all_sync(0xffffffffu, have && ok);
                const int qrow = r & 63;
                const bool store = qvalid && qrow < p.n_a[a];
                __nv_bfloat16* dst = p.out;
                if (store) {
                    const int t = p.slot_token[a * 64 + qrow];
                    dst += (size_t)(bh / p.H) * p.o0 + (size_t)(bh % p.H) * p.o1 + (size_t)t * p.o2;
                }
#pragma unroll 1
                for (int c0 = 0; c0 < D; c0 += 32) {
                    uint32_t o[32];
                    if (have_o) {
                        tmem_ld32(lane_base + kColO + c0, o);
                    } else {
#pragma unroll
                        for (int c = 0; c < 32; ++c) o[c] = 0u;
                    }
                    if (store) {
#pragma unroll
                        for (int c = 0; c < 16; ++c) {
                            const float x0 = o_scale > 0.0f ? __uint_as_float(o[2 * c]) * o_scale : 0.0f;
                            const float x1 = o_scale > 0.0f ? __uint_as_float(o[2 * c + 1]) * o_scale : 0.0f;
                            const __nv_bfloat162 b2 = __floats2bfloat162_rn(x0, x1);
                            o[c] = *reinterpret_cast<const uint32_t*>(&b2);
                        }
#pragma unroll
                        for (int v = 0; v < 4; ++v)
                            *reinterpret_cast<uint4*>(dst + c0 + 8 * v) =
                                make_uint4(o[4 * v], o[4 * v + 1], o[4 * v + 2], o[4 * v + 3]);
                    }
                }

            // the next item's first PV overwrites O: only after every load above
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bar_epi);
                mbar_arrive(&bar_infofree[k & 1]);
            }
            gstep += n_ent;
        }
        roles_done_barrier();
        if constexpr (!T16) setmaxnreg_inc<kRegLaunch>();
    }

    // ---- teardown: drain outstanding async work, then free tensor memory
    __syncthreads();
    if (warp == kMmaWarp && mma_issued) {
        tc_commit_w(&bar_drain);
        if (lane == 0 && !mbar_wait_drain(&bar_drain, 0, p.wait_ns)) atomicOr(p.status, DA2_DEV_TIMEOUT);
    }
    if (warp == kLoadWarp && lane == 0) {
        // every issued stage fill must have landed before the CTA exits
        for (uint32_t k = 0; k < loads_issued && k < (uint32_t)kStages; ++k) {
            const uint32_t g = loads_issued - 1 - k, st = g % kStages;
            if (!mbar_wait_drain(&bar_full[st], (g / kStages) & 1, p.wait_ns)) atomicOr(p.status, DA2_DEV_TIMEOUT);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// Shared memory of a CTA: the fixed layout plus the merged list.  Without the
// 16-bit path two CTAs share an SM (each at most ~113 KB and at least 80 KB, so
// that a third CTA never joins them: each holds 256 of the 512 tensor-memory
// columns for its lifetime); with it one CTA per SM.
template <int D, bool T16>
size_t attention_smem_bytes(int R) {
    const size_t need = Smem<D, T16>::list + (size_t)2 * R * sizeof(uint16_t);
    return (!T16 && need < 80 * 1024) ? 80 * 1024 : need;
}

// The warpgroups' register budgets (two CTAs per SM) assume the kernel is
// compiled for exactly kRegLaunch registers per thread; a different count
// would make the budget exchange wait forever, so the launch refuses it.
template <int D>
cudaError_t check_registers() {
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, attention_kernel<D, false>);
    if (e != cudaSuccess) return e;
    return fa.numRegs == (int)kRegLaunch ? cudaSuccess : cudaErrorInvalidKernelImage;
}

template <int D, bool T16>
cudaError_t launch_d(const AttnArgs& p, int items, cudaStream_t stream) {
    if constexpr (!T16) {
        const cudaError_t e = check_registers<D>();
        if (e != cudaSuccess) return e;
    }
    const int per_sm = T16 ? 1 : 2;
    const int grid = items < per_sm * p.num_sms ? items : per_sm * p.num_sms;
    const size_t smem = attention_smem_bytes<D, T16>(p.R);
    cudaError_t e = cudaFuncSetAttribute(attention_kernel<D, T16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attention_kernel<D, T16><<<grid, kThreads, smem, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention(const AttnArgs& p, cudaStream_t stream) {
    const int items = p.B * p.H * p.npairs;
    if (items == 0) return cudaSuccess;
    cudaError_t e = cudaMemsetAsync(p.work_counter, 0, sizeof(int), stream);
    if (e != cudaSuccess) return e;
    // the 16-bit phase runs when the prepared operands include the bf16 tiles
    const bool t16 = p.q16 != nullptr;
    if (p.d == 64) return t16 ? launch_d<64, true>(p, items, stream) : launch_d<64, false>(p, items, stream);
    return t16 ? launch_d<128, true>(p, items, stream) : launch_d<128, false>(p, items, stream);
}

}  // namespace da2

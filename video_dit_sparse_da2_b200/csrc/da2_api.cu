// da2_api.cu -- the extern "C" boundary of libda2 (declared in include/da2.h).
// Argument checks, the handle with its partition tables, buffer sizes, and
// the kernel launches of the three steps of "DraftAttention2"'s hot path.
#include <cstdio>
#include <cstring>
#include <new>
#include <vector>

#include "../../include/da2.h"
#include "da2_common.cuh"
#include "da2_kernels.h"
#include "da2_partition.h"

struct da2_ctx {
    da2_shape shape{};
    int Rf = 0, R = 0, N = 0, Npad = 0;  // R: all blocks (video, then prefix)
    int Rv = 0, Rp = 0;                    // video blocks, prefix blocks
    int device = 0, num_sms = 0;
    std::vector<int32_t> slot_token, n_a;  // host copies
    int32_t* d_slot_token = nullptr;       // [Npad]
    int32_t* d_n_a = nullptr;              // [R]
    int32_t* d_pairs = nullptr;            // [npairs][2] query blocks sharing an attention tile (-1: none)
    int npairs = 0;
    unsigned* d_status = nullptr;          // kernel status word
    int* d_work = nullptr;                 // attention work counter
    unsigned long long wait_ns = DA2_WAIT_NS_DEFAULT;  // limit of the kernels' bounded waits
};

namespace {

thread_local char g_cuda_error[256] = "";

int cuda_fail(cudaError_t e) {
    std::snprintf(g_cuda_error, sizeof(g_cuda_error), "%s: %s", cudaGetErrorName(e), cudaGetErrorString(e));
    return DA2_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool prepared_ok(const da2_prepared* p) {
    if (!p) return false;
    const void* ptrs[] = {p->desc, p->q8, p->k8, p->v8, p->q4, p->k4, p->v4, p->sfq, p->sfk, p->sfv, p->scale, p->vmax};
    for (const void* q : ptrs)
        if (!q || !aligned16(q)) return false;
    // the 16-bit operands: all three or none
    const bool any16 = p->q16 || p->k16 || p->v16, all16 = p->q16 && p->k16 && p->v16;
    if (any16 && (!all16 || !aligned16(p->q16) || !aligned16(p->k16) || !aligned16(p->v16))) return false;
    // the INT8 QK^T operands: all three or none
    const bool anyi = p->q8i || p->k8i || p->si8, alli = p->q8i && p->k8i && p->si8;
    if (anyi && (!alli || !aligned16(p->q8i) || !aligned16(p->k8i) || !aligned16(p->si8))) return false;
    return true;
}

bool budget_ok(const da2_budget* b) {
    return b && b->bp_fp8 >= 0 && b->bp_fp4 >= 0 && b->bp_fp16 >= 0 &&
           (long long)b->bp_fp16 + b->bp_fp8 + b->bp_fp4 <= 10000 && b->lambda >= 0.0 && b->lambda <= 1.0 &&
           (b->per_row == 0 || b->per_row == 1);
}

bool plan_ok(const da2_plan_bufs* p) {
    if (!p) return false;
    const void* ptrs[] = {p->prec, p->cnt, p->off, p->kidx, p->A, p->scratch};
    for (const void* q : ptrs)
        if (!q || !aligned16(q)) return false;
    return true;
}

}  // namespace

namespace da2 {
int handle_device(const da2_ctx* h) { return h->device; }
int record_cuda_error(cudaError_t e) { return cuda_fail(e); }
}  // namespace da2

extern "C" {

const char* da2_status_string(int status) {
    switch (status) {
        case DA2_OK: return "ok";
        case DA2_ERR_ARG: return "invalid argument";
        case DA2_ERR_ARCH: return "device is not sm_100 (B200)";
        case DA2_ERR_CUDA: return "CUDA error";
        case DA2_ERR_TIMEOUT: return "a bounded device-side wait gave up";
        default: return "unknown status";
    }
}

const char* da2_last_cuda_error(void) { return g_cuda_error; }

int da2_create(const da2_shape* s, da2_handle* out) {
    if (!s || !out) return DA2_ERR_ARG;
    *out = nullptr;
    if (s->B <= 0 || s->H <= 0 || s->F <= 0 || s->Hv <= 0 || s->Wv <= 0) return DA2_ERR_ARG;
    if (s->d != 64 && s->d != 128) return DA2_ERR_ARG;
    if (s->C != 64) return DA2_ERR_ARG;
    if (s->P < 0 || s->P > (1 << 20)) return DA2_ERR_ARG;
    const long long n = (long long)s->Hv * s->Wv;
    const long long Rf = (n + 63) / 64, R = Rf * s->F + (s->P + 63) / 64;
    if (R > 4096 || (long long)s->B * s->H * R * R > (1ll << 40)) return DA2_ERR_ARG;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    cudaDeviceProp prop;
    if ((e = cudaGetDeviceProperties(&prop, dev)) != cudaSuccess) return cuda_fail(e);
    if (prop.major != 10) return DA2_ERR_ARCH;

    da2::FramePartition part;
    if (!da2::build_partition(s->Hv, s->Wv, 64, &part)) return DA2_ERR_ARG;
    da2_ctx* h = new (std::nothrow) da2_ctx();
    if (!h) return DA2_ERR_CUDA;
    h->shape = *s;
    h->Rf = part.Rf;
    h->Rv = s->F * part.Rf;
    h->Rp = (s->P + 63) / 64;
    h->R = h->Rv + h->Rp;
    h->N = s->P + s->F * (int)n;
    h->Npad = 64 * h->R;
    h->device = dev;
    h->num_sms = prop.multiProcessorCount;
    h->slot_token.assign(h->Npad, -1);
    h->n_a.assign(h->R, 0);
    // video tokens follow the P prefix tokens; the prefix blocks (64
    // consecutive prefix tokens each) follow the video blocks
    for (int f = 0; f < s->F; ++f) {
        for (int j = 0; j < part.Rf; ++j) h->n_a[f * part.Rf + j] = part.size[j];
        for (long long c = 0; c < n; ++c) {
            const int a = f * part.Rf + part.region[c];
            h->slot_token[(size_t)a * 64 + part.slot[c]] = (int32_t)(s->P + f * n + c);
        }
    }
    for (int i = 0; i < h->Rp; ++i) {
        const int a = h->Rv + i, cnt = s->P - 64 * i < 64 ? s->P - 64 * i : 64;
        h->n_a[a] = cnt;
        for (int j = 0; j < cnt; ++j) h->slot_token[(size_t)a * 64 + j] = 64 * i + j;
    }
    // Query blocks that share one 128-row attention tile: block j of frame 2f
    // with block j of frame 2f + 1 (the same patch one frame later, whose key
    // lists are most alike in video, so the tile's merged list is shortest);
    // the blocks of a last, unpaired frame and the prefix blocks pair with
    // their successors.
    std::vector<int32_t> pairs;
    for (int f = 0; f + 1 < s->F; f += 2)
        for (int j = 0; j < part.Rf; ++j) {
            pairs.push_back(f * part.Rf + j);
            pairs.push_back((f + 1) * part.Rf + j);
        }
    auto successive = [&](int base, int n) {
        for (int i = 0; i < n; i += 2) {
            pairs.push_back(base + i);
            pairs.push_back(i + 1 < n ? base + i + 1 : -1);
        }
    };
    if (s->F % 2) successive((s->F - 1) * part.Rf, part.Rf);
    successive(h->Rv, h->Rp);
    h->npairs = (int)(pairs.size() / 2);
    if ((e = cudaMalloc(&h->d_slot_token, sizeof(int32_t) * h->Npad)) != cudaSuccess ||
        (e = cudaMalloc(&h->d_n_a, sizeof(int32_t) * h->R)) != cudaSuccess ||
        (e = cudaMalloc(&h->d_pairs, sizeof(int32_t) * pairs.size())) != cudaSuccess ||
        (e = cudaMemcpy(h->d_pairs, pairs.data(), sizeof(int32_t) * pairs.size(), cudaMemcpyHostToDevice)) !=
            cudaSuccess ||
        (e = cudaMalloc(&h->d_status, sizeof(unsigned))) != cudaSuccess ||
        (e = cudaMalloc(&h->d_work, sizeof(int))) != cudaSuccess ||
        (e = cudaMemcpy(h->d_slot_token, h->slot_token.data(), sizeof(int32_t) * h->Npad, cudaMemcpyHostToDevice)) !=
            cudaSuccess ||
        (e = cudaMemcpy(h->d_n_a, h->n_a.data(), sizeof(int32_t) * h->R, cudaMemcpyHostToDevice)) != cudaSuccess ||
        (e = cudaMemset(h->d_status, 0, sizeof(unsigned))) != cudaSuccess) {
        da2_destroy(h);
        return cuda_fail(e);
    }
    *out = h;
    return DA2_OK;
}

int da2_partition(int F, int Hv, int Wv, int32_t* slot_token, int32_t* n_a) {
    if (F <= 0) return DA2_ERR_ARG;
    da2::FramePartition part;
    if (!da2::build_partition(Hv, Wv, 64, &part)) return DA2_ERR_ARG;
    const int R = F * part.Rf, n = Hv * Wv;
    if (slot_token)
        for (int i = 0; i < 64 * R; ++i) slot_token[i] = -1;
    for (int f = 0; f < F; ++f) {
        for (int j = 0; j < part.Rf; ++j)
            if (n_a) n_a[f * part.Rf + j] = part.size[j];
        if (slot_token)
            for (int c = 0; c < n; ++c)
                slot_token[(size_t)(f * part.Rf + part.region[c]) * 64 + part.slot[c]] = f * n + c;
    }
    return R;
}

int da2_destroy(da2_handle h) {
    if (!h) return DA2_OK;
    cudaFree(h->d_slot_token);
    cudaFree(h->d_n_a);
    cudaFree(h->d_pairs);
    cudaFree(h->d_status);
    cudaFree(h->d_work);
    delete h;
    return DA2_OK;
}

int da2_sizes(da2_handle h, da2_sizes_t* o) {
    if (!h || !o) return DA2_ERR_ARG;
    const size_t BH = (size_t)h->shape.B * h->shape.H, R = h->R, Rv = h->Rv, d = h->shape.d;
    std::memset(o, 0, sizeof(*o));
    o->R = h->R;
    o->Rf = h->Rf;
    o->Npad = h->Npad;
    o->Rv = h->Rv;
    o->Rp = h->Rp;
    o->desc = 4 * BH * R * d * sizeof(double);
    o->q8 = o->k8 = o->v8 = BH * R * 64 * d;
    o->q4 = o->k4 = o->v4 = BH * R * 32 * d;
    o->sfq = BH * R * 64 * (d / 16);
    o->sfk = o->sfv = BH * R * 512;
    o->scale = 6 * BH * R * sizeof(float);
    o->vmax = 2 * BH * sizeof(float);
    o->prec = BH * Rv * Rv;
    o->cnt = 3 * BH * R * sizeof(int32_t);
    o->off = BH * (R + 1) * sizeof(int64_t);
    o->kidx = BH * R * R * sizeof(uint16_t);
    o->A = BH * Rv * Rv * sizeof(double);
    o->plan_scratch = da2::plan_scratch_bytes((int)BH, (int)Rv, h->shape.d);
    o->q16 = o->k16 = o->v16 = BH * R * 128 * d;
    o->q8i = o->k8i = BH * R * 64 * d;
    o->si8 = 2 * BH * R * sizeof(float);
    return DA2_OK;
}

int da2_list_bytes(da2_handle h, const da2_budget* budget, size_t* bytes) {
    if (!h || !bytes || !budget_ok(budget)) return DA2_ERR_ARG;
    const size_t BH = (size_t)h->shape.B * h->shape.H;
    *bytes = BH *
             (size_t)da2::plan_kept_per_head(h->Rv, h->Rp, budget->bp_fp16, budget->bp_fp8, budget->bp_fp4,
                                             budget->per_row) *
             sizeof(uint16_t);
    return DA2_OK;
}

int da2_tables(da2_handle h, int32_t* slot_token, int32_t* n_a) {
    if (!h) return DA2_ERR_ARG;
    if (slot_token) std::memcpy(slot_token, h->slot_token.data(), sizeof(int32_t) * h->Npad);
    if (n_a) std::memcpy(n_a, h->n_a.data(), sizeof(int32_t) * h->R);
    return DA2_OK;
}

int da2_prepare(da2_handle h, const void* q, const void* k, const void* v, const int64_t strides[4],
                const da2_prepared* out, void* stream) {
    if (!h || !q || !k || !v || !strides || !prepared_ok(out)) return DA2_ERR_ARG;
    if (strides[3] != 1 || strides[2] % 8 || strides[1] % 8 || strides[0] % 8 || strides[2] < h->shape.d)
        return DA2_ERR_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v)) return DA2_ERR_ARG;
    da2::PrepareArgs a{};
    a.B = h->shape.B;
    a.H = h->shape.H;
    a.d = h->shape.d;
    a.R = h->R;
    a.Rv = h->Rv;
    a.q = static_cast<const __nv_bfloat16*>(q);
    a.k = static_cast<const __nv_bfloat16*>(k);
    a.v = static_cast<const __nv_bfloat16*>(v);
    a.s0 = strides[0];
    a.s1 = strides[1];
    a.s2 = strides[2];
    a.slot_token = h->d_slot_token;
    a.n_a = h->d_n_a;
    a.desc = out->desc;
    a.q8 = out->q8; a.k8 = out->k8; a.v8 = out->v8;
    a.q4 = out->q4; a.k4 = out->k4; a.v4 = out->v4;
    a.sfq = out->sfq; a.sfk = out->sfk; a.sfv = out->sfv;
    a.q16 = out->q16; a.k16 = out->k16; a.v16 = out->v16;
    a.q8i = out->q8i; a.k8i = out->k8i; a.si8 = out->si8;
    a.scale = out->scale;
    a.vmax = out->vmax;
    a.status = h->d_status;
    a.wait_ns = h->wait_ns;
    a.num_sms = h->num_sms;
    cudaError_t e = da2::launch_prepare(a, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? DA2_OK : cuda_fail(e);
}

int da2_plan(da2_handle h, const da2_prepared* prep, const da2_budget* budget, const da2_plan_bufs* plan,
             void* stream) {
    if (!h || !prepared_ok(prep) || !budget_ok(budget) || !plan_ok(plan)) return DA2_ERR_ARG;
    da2::PlanArgs a{};
    a.BH = h->shape.B * h->shape.H;
    a.R = h->Rv;   // the ranking covers the video blocks
    a.Rt = h->R;   // lists, counts and prepared operands cover every block
    a.Rp = h->Rp;
    a.d = h->shape.d;
    a.bp16 = budget->bp_fp16;
    a.bp8 = budget->bp_fp8;
    a.bp4 = budget->bp_fp4;
    a.lambda = budget->lambda;
    a.per_row = budget->per_row;
    a.desc = prep->desc;
    a.A = plan->A;
    a.prec = plan->prec;
    a.cnt = plan->cnt;
    a.off = reinterpret_cast<long long*>(plan->off);
    a.kidx = plan->kidx;
    a.status = h->d_status;
    a.num_sms = h->num_sms;
    a.wait_ns = h->wait_ns;
    da2::plan_carve_scratch(&a, plan->scratch);
    cudaError_t e = da2::launch_plan(a, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? DA2_OK : cuda_fail(e);
}

int da2_attention(da2_handle h, const da2_prepared* prep, const da2_plan_bufs* plan, void* out,
                  const int64_t out_strides[4], void* stream) {
    if (!h || !prepared_ok(prep) || !plan_ok(plan) || !out || !out_strides) return DA2_ERR_ARG;
    if (out_strides[3] != 1 || out_strides[2] % 8 || out_strides[1] % 8 || out_strides[0] % 8 ||
        out_strides[2] < h->shape.d || !aligned16(out))
        return DA2_ERR_ARG;
    da2::AttnArgs a{};
    a.B = h->shape.B;
    a.H = h->shape.H;
    a.d = h->shape.d;
    a.R = h->R;
    a.N = h->N;
    a.slot_token = h->d_slot_token;
    a.n_a = h->d_n_a;
    a.q8 = prep->q8; a.k8 = prep->k8; a.v8 = prep->v8;
    a.q4 = prep->q4; a.k4 = prep->k4; a.v4 = prep->v4;
    a.sfq = prep->sfq; a.sfk = prep->sfk; a.sfv = prep->sfv;
    a.q16 = prep->q16; a.k16 = prep->k16; a.v16 = prep->v16;
    a.q8i = prep->q8i; a.k8i = prep->k8i; a.si8 = prep->si8;
    a.scale = prep->scale;
    a.vmax = prep->vmax;
    a.cnt = plan->cnt;
    a.off = reinterpret_cast<const long long*>(plan->off);
    a.kidx = plan->kidx;
    a.pairs = h->d_pairs;
    a.npairs = h->npairs;
    a.out = static_cast<__nv_bfloat16*>(out);
    a.o0 = out_strides[0];
    a.o1 = out_strides[1];
    a.o2 = out_strides[2];
    a.status = h->d_status;
    a.work_counter = h->d_work;
    a.num_sms = h->num_sms;
    a.wait_ns = h->wait_ns;
    cudaError_t e = da2::launch_attention(a, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? DA2_OK : cuda_fail(e);
}

int da2_set_wait_limit(da2_handle h, uint64_t limit_ns) {
    if (!h) return DA2_ERR_ARG;
    h->wait_ns = limit_ns ? (unsigned long long)limit_ns : DA2_WAIT_NS_DEFAULT;
    return DA2_OK;
}

int da2_selftest_wait_timeout(da2_handle h, uint64_t limit_ns, void* stream) {
    if (!h || limit_ns == 0 || limit_ns > 1000000000ull) return DA2_ERR_ARG;
    cudaError_t e = da2::launch_wait_selftest(h->d_status, limit_ns, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? DA2_OK : cuda_fail(e);
}

int da2_check_device_status(da2_handle h, void* stream) {
    if (!h) return DA2_ERR_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    unsigned st = 0;
    cudaError_t e = cudaMemcpyAsync(&st, h->d_status, sizeof(unsigned), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e == cudaSuccess) e = cudaMemsetAsync(h->d_status, 0, sizeof(unsigned), s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e);
    if (st & 1u) return DA2_ERR_TIMEOUT;
    if (st & 2u) return DA2_ERR_ARG;
    return DA2_OK;
}

}  // extern "C"

// da2_kernels.h -- launch interfaces of the DraftAttention2 kernels (internal).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

struct da2_ctx;

namespace da2 {

struct PrepareArgs {
    int B, H, d, R;            // R: every block (video, then prefix)
    int Rv;                    // video blocks (the V maxima cover these)
    const __nv_bfloat16 *q, *k, *v;
    long long s0, s1, s2;      // element strides of batch, head, token
    const int32_t* slot_token; // [64 R] token of each slot, -1 = padding
    const int32_t* n_a;        // [R]
    double* desc;
    uint8_t *q8, *k8, *v8, *q4, *k4, *v4, *sfq, *sfk, *sfv;
    uint8_t *q16, *k16, *v16;    // bf16 tiles of the 16-bit path, or all null
    int8_t *q8i, *k8i;           // INT8 tiles of Q and K, or null
    float* si8;                  // [2][BH][R] their tile scales, or null
    float* scale;
    float* vmax;
    unsigned* status;            // handle status word (bounded waits)
    unsigned long long wait_ns;  // limit of every bounded device-side wait
    int num_sms;
};
cudaError_t launch_prepare(const PrepareArgs& p, cudaStream_t stream);

// Per head and per quota target, the state of the radix selection of the
// T-th largest 96-bit key (A bits : ~pair index).
struct __align__(16) SelectTarget {
    unsigned long long p_hi;  // selected prefix, left aligned in 96 bits
    unsigned int p_lo;
    int nbits;                // bits of the key already fixed
    long long need;           // rank still sought inside the current prefix (1-based)
    int unique;               // the current prefix holds exactly one key: record it next pass
    int found;                // that key was recorded (the pass's scan then marks the target done)
    int done;                 // threshold known (or no threshold: none)
    int none;                 // T == 0: nothing gets this precision or better
    long long matches;        // keys that match the current prefix
    unsigned long long key_hi;
    unsigned int key_lo;
};

struct PlanArgs {
    int BH, R, d;            // R: video blocks (draft map, ranking, prec, A)
    int Rt, Rp;              // every block (Rv + Rp prefix blocks): descriptors, counts, lists
    int bp16, bp8, bp4;
    double lambda;
    int per_row;             // 1: quotas and ranking per query block instead of per head
    const double* desc;      // [4][BH][R][d]
    double* A;               // [BH][R][R] (first holds the average-branch logits)
    double* Lmax;            // [BH][R][R] max-branch logits (scratch)
    unsigned long long* abits_minmax;  // [BH][2] (scratch)
    SelectTarget* sel;       // [BH][3] (scratch): 16-bit, 8-bit, kept cuts
    unsigned int* hist;      // [BH][3][4096] (scratch)
    unsigned int* done_count;  // [BH] finished histogram CTAs of the current pass (scratch)
    int* cand_n;              // [BH] keys in the head's selection candidate list (scratch; the
                              //   list itself sits in the head's Lmax rows, dead after the softmax)
    int* cand_state;          // [BH] 0 no list, 1 list collected (later passes read it)
    uint8_t* prec;           // [BH][R][R]
    int32_t* cnt;            // [3][BH][R]: 8-bit, 4-bit, 16-bit counts
    long long* off;          // [BH][R+1] list offsets (positions in kidx)
    uint16_t* kidx;          // [BH * kept per head] compact lists
    unsigned* status;
    int num_sms;             // multiprocessors of the device (grid sizing)
    unsigned long long wait_ns;  // limit of the bounded device waits
    // max-pool branch from exact integer tensor-core products (scratch):
    int8_t* mx_tiles;        // [2][BH][Rpad/128][3 parts][128 * d] split descriptors, K-major
    int* mx_e0;              // [2][BH][Rpad] smallest exponent of each block
    uint8_t* mx_ok;          // [2][BH][Rpad] block inside the exact range
    int* mx_fail;            // [1 + 2 BH Rpad]: count, then (t BH + bh) Rpad + r of each block outside it
    int mx_rpad;             // R rounded up to 128
};
size_t plan_scratch_bytes(int BH, int R, int d);
size_t mx_scratch_bytes(int BH, int R, int d);
void mx_carve(PlanArgs* p, char* c);
cudaError_t launch_max_logits(const PlanArgs& p, double rd, cudaStream_t stream);
// Kept pairs of one head under a budget (the length of its part of kidx).
long long plan_kept_per_head(int Rv, int Rp, int bp16, int bp8, int bp4, int per_row);
void plan_carve_scratch(PlanArgs* p, void* scratch);
cudaError_t launch_plan(const PlanArgs& p, cudaStream_t stream);

struct AttnArgs {
    int B, H, d, R, N;
    const int32_t* slot_token;  // [64 R]
    const int32_t* n_a;         // [R]
    const int32_t* pairs;       // [npairs][2] query blocks of each work item's tile (second -1: none)
    int npairs;
    const uint8_t *q8, *k8, *v8, *q4, *k4, *v4, *sfq, *sfk, *sfv;
    const uint8_t *q16, *k16, *v16;  // bf16 tiles of the 16-bit path, or all null
    const int8_t *q8i, *k8i;         // INT8 Q/K tiles: the 8-bit phase's QK^T in INT8, or null
    const float* si8;                // [2][BH][R] their tile scales
    const float* scale;  // [6][BH][R]
    const float* vmax;   // [2][BH]
    const int32_t* cnt;  // [3][BH][R]: 8-bit, 4-bit, 16-bit counts
    const long long* off;  // [BH][R+1]
    const uint16_t* kidx;  // compact lists at off
    __nv_bfloat16* out;
    long long o0, o1, o2;  // element strides of the output
    unsigned* status;
    int* work_counter;  // item counter of the persistent CTAs (zeroed per launch)
    int num_sms;
    unsigned long long wait_ns;  // limit of every bounded device-side wait
};
cudaError_t launch_attention(const AttnArgs& p, cudaStream_t stream);

// Failure-path self-test: one CTA waits, with the given limit, on an mbarrier
// that nothing arrives on (see da2_selftest_wait_timeout in da2.h).
cudaError_t launch_wait_selftest(unsigned* status, unsigned long long limit_ns, cudaStream_t stream);

// Helpers of the C ABI used by its other translation units.
int handle_device(const struct ::da2_ctx* h);
int record_cuda_error(cudaError_t e);

}  // namespace da2

// decode.cu -- the KDA recurrent decode step (one token per sequence).
//
// Kimi Linear paper notes (paper-notes-site): section 2 gives the recurrence,
// section 3 the fused recurrent mode for short queries, which keeps only the
// recurrent state.  Per (sequence, head):
//     a = exp(g);  S' = Diag(a) S;  u = beta (v - S'^T k);
//     S = S' + k u^T;  o = S^T q = S'^T q + (q.k) u
// The state (dk x dv fp32, 64 KiB at d = 128) is read once and written once;
// everything else is small.  The kernel is HBM-bound: one CTA streams one
// state with 128-bit loads/stores, keeps it in registers while two column
// reductions (k^T S', q^T S') run, and writes it back.
//
// Mapping (NT = 256 threads): thread t owns the float4 column group
// t % (DV/4) of rows [rg*RPT, rg*RPT + RPT), rg = t / (DV/4).  At
// DK = DV = 128 a warp covers one full 512-byte row per load instruction.
// Column sums over rows: in-thread over RPT rows, then across row groups
// through shared memory.
#include "common.cuh"
#include "kernels.h"

namespace kda {

template <int LO, int HI, int W>
__device__ __forceinline__ float tree_sum(const float (*red)[W], int col) {
    if constexpr (HI - LO == 1) {
        return red[LO][col];
    } else {
        constexpr int MID = (LO + HI) / 2;
        return tree_sum<LO, MID>(red, col) + tree_sum<MID, HI>(red, col);
    }
}

template <int DK, int DV, typename Tin, bool PRO>
__global__ void __launch_bounds__(256, 2)
decode_step_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k,
                   const Tin *__restrict__ v, const float *__restrict__ g,
                   const float *__restrict__ beta, float *__restrict__ state,
                   const int32_t *__restrict__ slots, int num_slots, int H,
                   Tin *__restrict__ out, int *__restrict__ err, Prologue pro)
{
    constexpr int NT = 256;
    constexpr int C4 = DV / 4;       // float4 groups per row
    constexpr int RG = NT / C4;      // row groups
    constexpr int RPT = DK / RG;     // rows per thread
    static_assert(NT % C4 == 0 && DK % RG == 0, "bad decode tiling");

    const size_t nh = blockIdx.x;    // flattened (sequence, head)
    const int tid = threadIdx.x;
    const int c4 = tid % C4;
    const int rg = tid / C4;
    // state entry: slots[n] of a [num_slots, H] pool, or nh itself
    size_t sidx = nh;
    if (slots) {
        const int n = (int)(nh / H), h = (int)(nh - (size_t)n * H);
        const int slot = slots[n];
        if (slot < 0 || slot >= num_slots) {
            if (tid == 0) set_device_error(err, kErrBadSlot);
            return;
        }
        sidx = (size_t)slot * H + h;
    }

    __shared__ float ks[DK], qs[DK], as_[DK];
    __shared__ __align__(16) float red_k[RG][DV + 4];
    __shared__ __align__(16) float red_q[RG][DV + 4];
    __shared__ __align__(16) float us[DV];
    __shared__ float qk_part[NT / 32], kk_part[NT / 32], qq_part[NT / 32];

    // 1. Issue every state load first (64 KiB in flight per CTA at d=128).
    float4 *Sp = reinterpret_cast<float4 *>(state + sidx * (size_t)(DK * DV));
    float4 s[RPT];
#pragma unroll
    for (int r = 0; r < RPT; ++r) s[r] = ld_stream(Sp + (size_t)(rg * RPT + r) * C4 + c4);

    // 2. Token vectors; alpha = exp(g).
    float qk = 0.f, kk = 0.f, qq = 0.f;
    if (tid < DK) {
        const float kv = to_f(k[nh * DK + tid]);
        const float qv = to_f(q[nh * DK + tid]);
        ks[tid] = kv;
        qs[tid] = qv;
        as_[tid] = expf(g[nh * DK + tid]);
        qk = kv * qv;
        if (PRO) { kk = kv * kv; qq = qv * qv; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        qk += __shfl_xor_sync(0xffffffffu, qk, o);
        if (PRO) {
            kk += __shfl_xor_sync(0xffffffffu, kk, o);
            qq += __shfl_xor_sync(0xffffffffu, qq, o);
        }
    }
    if ((tid & 31) == 0) {
        qk_part[tid >> 5] = qk;
        if (PRO) { kk_part[tid >> 5] = kk; qq_part[tid >> 5] = qq; }
    }
    __syncthreads();
    // prologue factors: k <- sk k, q <- sq q
    float sk = 1.f, sq = 1.f;
    if (PRO) {
        if (pro.flags & kProQkL2Norm) {
            float ka = 0.f, qa = 0.f;
#pragma unroll
            for (int w = 0; w < NT / 32; ++w) { ka += kk_part[w]; qa += qq_part[w]; }
            sk = inv_norm(ka);
            sq = inv_norm(qa);
        }
        sq *= pro.q_scale;
    }

    // 3. S' = Diag(a) S and the per-thread partial column sums.
    float pk[4] = {0.f, 0.f, 0.f, 0.f}, pq[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
        const int row = rg * RPT + r;
        const float a = as_[row];
        float kr = ks[row], qr = qs[row];
        if (PRO) { kr *= sk; qr *= sq; }
        s[r].x *= a; s[r].y *= a; s[r].z *= a; s[r].w *= a;
        pk[0] = __fmaf_rn(kr, s[r].x, pk[0]); pk[1] = __fmaf_rn(kr, s[r].y, pk[1]);
        pk[2] = __fmaf_rn(kr, s[r].z, pk[2]); pk[3] = __fmaf_rn(kr, s[r].w, pk[3]);
        pq[0] = __fmaf_rn(qr, s[r].x, pq[0]); pq[1] = __fmaf_rn(qr, s[r].y, pq[1]);
        pq[2] = __fmaf_rn(qr, s[r].z, pq[2]); pq[3] = __fmaf_rn(qr, s[r].w, pq[3]);
    }
    reinterpret_cast<float4 *>(&red_k[rg][0])[c4] = make_float4(pk[0], pk[1], pk[2], pk[3]);
    reinterpret_cast<float4 *>(&red_q[rg][0])[c4] = make_float4(pq[0], pq[1], pq[2], pq[3]);
    __syncthreads();

    // 4. Finish the column sums; u = beta (v - S'^T k); o = S'^T q + (q.k) u.
    if (tid < DV) {
        // row groups summed as a balanced tree in row-group order (the same
        // order as the warp butterfly of the L-token kernel, decode_pipe.cu)
        const float kS = tree_sum<0, RG>(red_k, tid), qS = tree_sum<0, RG>(red_q, tid);
        float qk_all = 0.f;
#pragma unroll
        for (int w = 0; w < NT / 32; ++w) qk_all += qk_part[w];
        float b = beta[nh];
        if (PRO) {
            qk_all *= sk * sq;
            if (pro.flags & kProBetaSigmoid) b = sigmoid_f(b);
        }
        const float u = b * (to_f(v[nh * DV + tid]) - kS);
        us[tid] = u;
        out[nh * DV + tid] = from_f<Tin>(__fmaf_rn(qk_all, u, qS));
    }
    __syncthreads();

    // 5. S = S' + k u^T, written once.
    const float4 u4 = reinterpret_cast<const float4 *>(us)[c4];
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
        float kr = ks[rg * RPT + r];
        if (PRO) kr *= sk;
        float4 o4 = s[r];
        o4.x = __fmaf_rn(kr, u4.x, o4.x); o4.y = __fmaf_rn(kr, u4.y, o4.y);
        o4.z = __fmaf_rn(kr, u4.z, o4.z); o4.w = __fmaf_rn(kr, u4.w, o4.w);
        st_stream(Sp + (size_t)(rg * RPT + r) * C4 + c4, o4);
    }
}

template <int DK, int DV, typename Tin>
static cudaError_t launch_decode_t(const void *q, const void *k, const void *v,
                                   const float *g, const float *beta, float *state,
                                   const int32_t *slots, int num_slots, int H, void *out, int NH,
                                   int *err, Prologue pro, cudaStream_t st)
{
    auto kern = (pro.flags != 0 || pro.q_scale != 1.f) ? decode_step_kernel<DK, DV, Tin, true>
                                                       : decode_step_kernel<DK, DV, Tin, false>;
    kern<<<NH, 256, 0, st>>>((const Tin *)q, (const Tin *)k, (const Tin *)v, g, beta, state, slots,
                             num_slots, H, (Tin *)out, err, pro);
    return cudaGetLastError();
}

template <typename Tin>
static cudaError_t launch_decode_d(const void *q, const void *k, const void *v,
                                   const float *g, const float *beta, float *state,
                                   const int32_t *slots, int num_slots, int H, void *out, int NH,
                                   int dk, int dv, int *err, Prologue pro, cudaStream_t st)
{
#define KDA_STEP(DK_, DV_)                                                                       \
    if (dk == DK_ && dv == DV_)                                                                  \
        return launch_decode_t<DK_, DV_, Tin>(q, k, v, g, beta, state, slots, num_slots, H, out, \
                                              NH, err, pro, st);
    KDA_STEP(128, 128)
    KDA_STEP(64, 64)
    KDA_STEP(128, 64)
    KDA_STEP(64, 128)
#undef KDA_STEP
    return cudaErrorInvalidValue;
}

cudaError_t launch_decode(const void *q, const void *k, const void *v, const float *g,
                          const float *beta, float *state, void *out, int NH, int dk,
                          int dv, bool bf16, Prologue pro, cudaStream_t st)
{
    if (NH == 0) return cudaSuccess;
    if (bf16)
        return launch_decode_d<__nv_bfloat16>(q, k, v, g, beta, state, nullptr, 0, 1, out, NH, dk,
                                              dv, nullptr, pro, st);
    return launch_decode_d<float>(q, k, v, g, beta, state, nullptr, 0, 1, out, NH, dk, dv, nullptr,
                                  pro, st);
}

cudaError_t launch_decode_slots(const void *q, const void *k, const void *v, const float *g,
                                const float *beta, float *pool, const int32_t *slots,
                                int num_slots, void *out, int N, int H, int dk, int dv, bool bf16,
                                int *err, Prologue pro, cudaStream_t st)
{
    if (N == 0) return cudaSuccess;
    // without slots, sequence n uses entry n: the plain layout
    if (bf16)
        return launch_decode_d<__nv_bfloat16>(q, k, v, g, beta, pool, slots, num_slots, H, out,
                                              N * H, dk, dv, err, pro, st);
    return launch_decode_d<float>(q, k, v, g, beta, pool, slots, num_slots, H, out, N * H, dk, dv,
                                  err, pro, st);
}

}  // namespace kda

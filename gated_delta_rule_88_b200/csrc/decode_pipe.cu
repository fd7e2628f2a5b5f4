// decode_pipe.cu -- the L-token KDA decode on a slot-indexed state pool,
// as a persistent pipelined kernel.
//
// Kimi Linear paper notes (paper-notes-site): section 2 gives the recurrence,
// section 3 the fused recurrent mode for queries of at most 64 tokens.  Per
// (sequence, head) and token:
//     a = exp(g);  S' = Diag(a) S;  u = beta (v - S'^T k);
//     S = S' + k u^T;  o = S^T q = S'^T q + (q.k) u
//
// The columns of S are independent given the token vectors: column c needs
// only k, q, a, beta and v_c.  So each warp owns DV/8 columns over all DK
// rows and runs the whole token loop without talking to the other warps; the
// column sums k^T S', q^T S' are an in-thread sum over the lane's rows plus a
// shuffle butterfly across the warp's row groups.  The token vectors (k, q,
// exp(g) after the optional prologue) are prepared once per block of TB
// tokens into shared memory, shared by the eight warps.
//
// Pipelining: CTAs are persistent (two per SM) and walk the (sequence, head)
// items with a grid stride.  While item j is computed from registers, the
// state of item j+1 arrives in shared memory by one bulk copy (no multicast),
// and the raw token rows of the next block arrive by cp.async, so the HBM
// stream and the arithmetic overlap.  States are written back from registers
// with streaming stores.
//
// Lane mapping (warp w, lane = rgl * C4W + cg): columns w*CW + 4cg .. +3,
// rows rgl*RPT .. rgl*RPT + RPT - 1.  At DK = DV = 128: CW = 16, C4W = 4,
// RGW = 8 row groups, RPT = 16 rows, 64 state floats per thread.
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace kda {
using namespace sm100;
namespace {

template <int DK, int DV, typename Tin>
struct PipeCfg {
    static constexpr int NW = 8, NT = NW * 32;
    static constexpr int CW = DV / NW;          // columns per warp
    static constexpr int C4W = CW / 4;          // lanes across a warp's columns
    static constexpr int RGW = 32 / C4W;        // row groups per warp
    static constexpr int RPT = DK / RGW;        // rows per lane
    static constexpr int RS = RPT + 4;          // padded row-group stride (conflict-free LDS.128)
    static constexpr int VEC = RGW * RS;        // floats per staged vector
    static constexpr int TB = sizeof(Tin) == 2 ? 8 : 4;   // tokens per staged block
    static constexpr int RL = DK / 32;          // rows per lane when preparing a token
    // raw token row in shared memory: k, q, v (Tin), g (fp32), beta (16-byte slot)
    static constexpr int RK = DK * (int)sizeof(Tin), RV = DV * (int)sizeof(Tin), RG = DK * 4;
    static constexpr int RAW_TOK = 2 * RK + RV + RG + 16;
    static constexpr int CPT = (2 * RK + RV + RG) / 16 + 1;    // cp.async pieces per token
    static constexpr int STATE_BYTES = DK * DV * 4;
    static constexpr int OFF_RAW = STATE_BYTES;
    static constexpr int RAW_BYTES = TB * RAW_TOK;
    static constexpr int OFF_STG = OFF_RAW + 2 * RAW_BYTES;
    static constexpr int STG_TOK = (3 * VEC + 4) * 4;          // k^, q^, a, then (qk, beta)
    static constexpr int OFF_BAR = OFF_STG + TB * STG_TOK;
    static constexpr int BYTES = OFF_BAR + 16;
    static_assert(CW % 4 == 0 && 32 % C4W == 0 && DK % RGW == 0 && RPT % 4 == 0, "tiling");
    static_assert(RAW_TOK % 16 == 0 && STG_TOK % 16 == 0 && OFF_STG % 16 == 0, "alignment");
    static_assert(DK % 32 == 0 && TB <= NW, "token preparation: one warp per token");
};

__device__ __forceinline__ void cp_async4(void *smem_dst, const void *gmem_src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(smem_u32(smem_dst)),
                 "l"(gmem_src));
}

__device__ __forceinline__ void load4(const float *p, float (&x)[4]) {
    const float4 t = *reinterpret_cast<const float4 *>(p);
    x[0] = t.x; x[1] = t.y; x[2] = t.z; x[3] = t.w;
}
__device__ __forceinline__ void load4(const __nv_bfloat16 *p, float (&x)[4]) {
    const uint2 t = *reinterpret_cast<const uint2 *>(p);
    const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162 *>(&t.x);
    const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162 *>(&t.y);
    x[0] = __low2float(lo); x[1] = __high2float(lo); x[2] = __low2float(hi); x[3] = __high2float(hi);
}
__device__ __forceinline__ void store4(float *p, const float (&x)[4]) {
    *reinterpret_cast<float4 *>(p) = make_float4(x[0], x[1], x[2], x[3]);
}
__device__ __forceinline__ void store4(__nv_bfloat16 *p, const float (&x)[4]) {
    uint2 t;
    t.x = pack_bf16(x[0], x[1]);
    t.y = pack_bf16(x[2], x[3]);
    *reinterpret_cast<uint2 *>(p) = t;
}
__device__ __forceinline__ float comp(const float4 &v, int i) {
    return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

}  // namespace

template <int DK, int DV, typename Tin, bool PRO>
__global__ void __launch_bounds__(256, 2)
decode_pipe_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k,
                   const Tin *__restrict__ v, const float *__restrict__ g,
                   const float *__restrict__ beta, float *__restrict__ pool,
                   const int32_t *__restrict__ slots, int num_slots, Tin *__restrict__ out,
                   int N, int H, int L, int *__restrict__ err, Prologue pro)
{
    using C = PipeCfg<DK, DV, Tin>;
    extern __shared__ __align__(128) unsigned char smem[];
    float *st_s = reinterpret_cast<float *>(smem);
    unsigned char *raw = smem + C::OFF_RAW;
    unsigned char *stg = smem + C::OFF_STG;
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);

    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const int cg = lane % C::C4W, rgl = lane / C::C4W;
    const int col0 = w * C::CW + cg * 4;
    const int items = N * H;
    const int nblk = (L + C::TB - 1) / C::TB;

    // The next item at or after `it` (grid stride) whose slot is valid; -1 if
    // none.  Every thread walks the same items, so the answer is uniform.
    auto next_valid = [&](int it) -> int {
        for (; it < items; it += gridDim.x) {
            const int n = it / H;
            const int s = slots ? slots[n] : n;
            if (s >= 0 && s < num_slots) return it;
            if (tid == 0) set_device_error(err, kErrBadSlot);
        }
        return -1;
    };
    auto state_ptr = [&](int it) -> float * {
        const int n = it / H, h = it - n * H;
        const int s = slots ? slots[n] : n;
        return pool + ((size_t)s * H + h) * (size_t)(DK * DV);
    };
    auto token_row = [&](int it, int l) -> size_t {
        const int n = it / H, h = it - n * H;
        return ((size_t)n * L + l) * H + h;
    };
    // Raw rows of block (it, tb) into raw buffer `buf` (cp.async, one group).
    auto issue_raw = [&](int it, int tb, int buf) {
        const int nt = min(C::TB, L - tb * C::TB);
        unsigned char *dst0 = raw + buf * C::RAW_BYTES;
        for (int c = tid; c < nt * C::CPT; c += C::NT) {
            const int t = c / C::CPT, r = c - t * C::CPT;
            const size_t row = token_row(it, tb * C::TB + t);
            unsigned char *dst = dst0 + t * C::RAW_TOK;
            if (r < C::RK / 16) {
                cp_async16(dst + r * 16, reinterpret_cast<const unsigned char *>(k + row * DK) + r * 16);
            } else if (r < 2 * C::RK / 16) {
                const int o = r * 16 - C::RK;
                cp_async16(dst + C::RK + o, reinterpret_cast<const unsigned char *>(q + row * DK) + o);
            } else if (r < (2 * C::RK + C::RV) / 16) {
                const int o = r * 16 - 2 * C::RK;
                cp_async16(dst + 2 * C::RK + o, reinterpret_cast<const unsigned char *>(v + row * DV) + o);
            } else if (r < C::CPT - 1) {
                const int o = r * 16 - 2 * C::RK - C::RV;
                cp_async16(dst + 2 * C::RK + C::RV + o,
                           reinterpret_cast<const unsigned char *>(g + row * DK) + o);
            } else {
                cp_async4(dst + 2 * C::RK + C::RV + C::RG, beta + row);
            }
        }
        cp_async_commit();
    };
    auto issue_state = [&](int it) {
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(bar, C::STATE_BYTES);
        bulk_g2s(st_s, state_ptr(it), C::STATE_BYTES, bar);
    };

    if (tid == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
    }
    __syncthreads();

    int cur = next_valid(blockIdx.x);
    if (cur < 0) return;
    if (tid == 0) issue_state(cur);
    issue_raw(cur, 0, 0);

    uint32_t phase = 0;
    int buf = 0;
    // The lane's state rows as column pairs (c0, c1) and (c2, c3): the
    // per-element work runs as packed fp32x2 operations (each half rounds
    // exactly like the scalar operation).
    float2 s0[C::RPT], s1[C::RPT];
    while (cur >= 0) {
        const int nxt = next_valid(cur + gridDim.x);
        for (int tb = 0; tb < nblk; ++tb) {
            cp_async_wait<0>();
            __syncthreads();     // raw[buf] landed; every warp is done with the previous block
            if (tb == 0) {
                const bool late = !mbar_wait(bar, phase);
                if (__syncthreads_or(late)) {
                    // the state copy did not arrive: report and stop this CTA
                    // (no further copies are issued; no cp.async is pending)
                    if (tid == 0) set_device_error(err, kErrWaitTimeout);
                    return;
                }
                phase ^= 1u;
#pragma unroll
                for (int i = 0; i < C::RPT; ++i) {
                    const float4 x = *reinterpret_cast<const float4 *>(st_s + (rgl * C::RPT + i) * DV + col0);
                    s0[i] = make_float2(x.x, x.y);
                    s1[i] = make_float2(x.z, x.w);
                }
            }
            const int nt = min(C::TB, L - tb * C::TB);
            // Prepare token w of the block: prologue, exp(g), padded layout.
            if (w < nt) {
                const unsigned char *rt = raw + buf * C::RAW_BYTES + w * C::RAW_TOK;
                const Tin *kr = reinterpret_cast<const Tin *>(rt);
                const Tin *qr = reinterpret_cast<const Tin *>(rt + C::RK);
                const float *gr = reinterpret_cast<const float *>(rt + 2 * C::RK + C::RV);
                // lane holds elements lane + 32 j; each 32-element slice is
                // summed by a butterfly, the slices in order
                float kv[C::RL], qv[C::RL];
                float kq = 0.f, kk = 0.f, qq = 0.f;
#pragma unroll
                for (int j = 0; j < C::RL; ++j) {
                    kv[j] = to_f(kr[lane + 32 * j]);
                    qv[j] = to_f(qr[lane + 32 * j]);
                    float pkq = kv[j] * qv[j], pkk = 0.f, pqq = 0.f;
                    if (PRO) { pkk = kv[j] * kv[j]; pqq = qv[j] * qv[j]; }
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) {
                        pkq += __shfl_xor_sync(0xffffffffu, pkq, o);
                        if (PRO) {
                            pkk += __shfl_xor_sync(0xffffffffu, pkk, o);
                            pqq += __shfl_xor_sync(0xffffffffu, pqq, o);
                        }
                    }
                    kq += pkq;
                    if (PRO) { kk += pkk; qq += pqq; }
                }
                float sk = 1.f, sq = 1.f;
                if (PRO) {
                    if (pro.flags & kProQkL2Norm) { sk = inv_norm(kk); sq = inv_norm(qq); }
                    sq *= pro.q_scale;
                }
                float *sv = reinterpret_cast<float *>(stg + w * C::STG_TOK);
#pragma unroll
                for (int j = 0; j < C::RL; ++j) {
                    const int r = lane + 32 * j;
                    const int idx = (r / C::RPT) * C::RS + r % C::RPT;
                    sv[idx] = PRO ? kv[j] * sk : kv[j];
                    sv[C::VEC + idx] = PRO ? qv[j] * sq : qv[j];
                    sv[2 * C::VEC + idx] = expf(gr[r]);
                }
                if (lane == 0) {
                    float b = *reinterpret_cast<const float *>(rt + 2 * C::RK + C::RV + C::RG);
                    if (PRO && (pro.flags & kProBetaSigmoid)) b = sigmoid_f(b);
                    sv[3 * C::VEC] = PRO ? kq * (sk * sq) : kq;
                    sv[3 * C::VEC + 1] = b;
                }
            }
            __syncthreads();     // staged vectors visible; the state buffer has been read
            if (tb == 0 && nxt >= 0 && tid == 0) issue_state(nxt);
            if (tb + 1 < nblk) issue_raw(cur, tb + 1, buf ^ 1);
            else if (nxt >= 0) issue_raw(nxt, 0, buf ^ 1);

            // Token steps of this block, per warp, on its columns.
            const unsigned char *rv0 = raw + buf * C::RAW_BYTES + 2 * C::RK;
            for (int t = 0; t < nt; ++t) {
                const float *sv = reinterpret_cast<const float *>(stg + t * C::STG_TOK);
                const float qk = sv[3 * C::VEC], b = sv[3 * C::VEC + 1];
                float vv[4];
                load4(reinterpret_cast<const Tin *>(rv0 + t * C::RAW_TOK) + col0, vv);
                // S' = Diag(a) S; partial column sums k^T S', q^T S' over the
                // lane's rows in row order
                float2 pk0 = make_float2(0.f, 0.f), pk1 = pk0, pq0 = pk0, pq1 = pk0;
#pragma unroll
                for (int i = 0; i < C::RPT; i += 4) {
                    const int idx = rgl * C::RS + i;
                    const float4 K = *reinterpret_cast<const float4 *>(sv + idx);
                    const float4 Q = *reinterpret_cast<const float4 *>(sv + C::VEC + idx);
                    const float4 A = *reinterpret_cast<const float4 *>(sv + 2 * C::VEC + idx);
#pragma unroll
                    for (int ii = 0; ii < 4; ++ii) {
                        const float a = comp(A, ii), kr = comp(K, ii), qr = comp(Q, ii);
                        const float2 a2 = make_float2(a, a), k2 = make_float2(kr, kr),
                                     q2 = make_float2(qr, qr);
                        s0[i + ii] = __fmul2_rn(s0[i + ii], a2);
                        s1[i + ii] = __fmul2_rn(s1[i + ii], a2);
                        pk0 = __ffma2_rn(k2, s0[i + ii], pk0);
                        pk1 = __ffma2_rn(k2, s1[i + ii], pk1);
                        pq0 = __ffma2_rn(q2, s0[i + ii], pq0);
                        pq1 = __ffma2_rn(q2, s1[i + ii], pq1);
                    }
                }
                // across the warp's row groups: a balanced tree in row-group
                // order (column pairs added as fp32x2, each half rounding like
                // the scalar add)
#pragma unroll
                for (int o = C::C4W; o < 32; o <<= 1) {
                    pk0 = __fadd2_rn(pk0, make_float2(__shfl_xor_sync(0xffffffffu, pk0.x, o),
                                                      __shfl_xor_sync(0xffffffffu, pk0.y, o)));
                    pk1 = __fadd2_rn(pk1, make_float2(__shfl_xor_sync(0xffffffffu, pk1.x, o),
                                                      __shfl_xor_sync(0xffffffffu, pk1.y, o)));
                    pq0 = __fadd2_rn(pq0, make_float2(__shfl_xor_sync(0xffffffffu, pq0.x, o),
                                                      __shfl_xor_sync(0xffffffffu, pq0.y, o)));
                    pq1 = __fadd2_rn(pq1, make_float2(__shfl_xor_sync(0xffffffffu, pq1.x, o),
                                                      __shfl_xor_sync(0xffffffffu, pq1.y, o)));
                }
                // u = beta (v - k^T S'), o = q^T S' + (q.k) u, per column pair
                const float2 b2 = make_float2(b, b), qk2 = make_float2(qk, qk);
                const float2 u01 = __fmul2_rn(b2, __fadd2_rn(make_float2(vv[0], vv[1]), make_float2(-pk0.x, -pk0.y)));
                const float2 u23 = __fmul2_rn(b2, __fadd2_rn(make_float2(vv[2], vv[3]), make_float2(-pk1.x, -pk1.y)));
                const float2 o01 = __ffma2_rn(qk2, u01, pq0), o23 = __ffma2_rn(qk2, u23, pq1);
                float ov[4] = {o01.x, o01.y, o23.x, o23.y};
                if (rgl == 0) store4(out + token_row(cur, tb * C::TB + t) * DV + col0, ov);
                // S = S' + k u^T
#pragma unroll
                for (int i = 0; i < C::RPT; i += 4) {
                    const float4 K = *reinterpret_cast<const float4 *>(sv + rgl * C::RS + i);
#pragma unroll
                    for (int ii = 0; ii < 4; ++ii) {
                        const float kr = comp(K, ii);
                        const float2 k2 = make_float2(kr, kr);
                        s0[i + ii] = __ffma2_rn(k2, u01, s0[i + ii]);
                        s1[i + ii] = __ffma2_rn(k2, u23, s1[i + ii]);
                    }
                }
            }
            buf ^= 1;
        }
        float4 *Sp = reinterpret_cast<float4 *>(state_ptr(cur));
#pragma unroll
        for (int i = 0; i < C::RPT; ++i)
            st_stream(Sp + ((rgl * C::RPT + i) * DV + col0) / 4,
                      make_float4(s0[i].x, s0[i].y, s1[i].x, s1[i].y));
        cur = nxt;
    }
}

namespace {

template <int DK, int DV, typename Tin, bool PRO>
cudaError_t launch_pipe(const void *q, const void *k, const void *v, const float *g,
                        const float *beta, float *pool, const int32_t *slots, int num_slots,
                        void *out, int N, int H, int L, int *err, Prologue pro, cudaStream_t st)
{
    using C = PipeCfg<DK, DV, Tin>;
    auto kern = decode_pipe_kernel<DK, DV, Tin, PRO>;
    // per device: the smem opt-in and the resident CTAs per SM x SMs
    static int grid_for[64] = {0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (grid_for[dev] == 0) {
        if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::BYTES)) != cudaSuccess)
            return e;
        int sms = 0, per_sm = 0;
        if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
        if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, C::NT, C::BYTES)) != cudaSuccess)
            return e;
        grid_for[dev] = sms * (per_sm > 0 ? per_sm : 1);
    }
    const int items = N * H;
    const int grid = items < grid_for[dev] ? items : grid_for[dev];
    kern<<<grid, C::NT, C::BYTES, st>>>((const Tin *)q, (const Tin *)k, (const Tin *)v, g, beta,
                                        pool, slots, num_slots, (Tin *)out, N, H, L, err, pro);
    return cudaGetLastError();
}

template <int DK, int DV, typename Tin>
cudaError_t launch_pipe_p(const void *q, const void *k, const void *v, const float *g,
                          const float *beta, float *pool, const int32_t *slots, int num_slots,
                          void *out, int N, int H, int L, int *err, Prologue pro, cudaStream_t st)
{
    if (pro.flags != 0 || pro.q_scale != 1.f)
        return launch_pipe<DK, DV, Tin, true>(q, k, v, g, beta, pool, slots, num_slots, out, N, H, L, err, pro, st);
    return launch_pipe<DK, DV, Tin, false>(q, k, v, g, beta, pool, slots, num_slots, out, N, H, L, err, pro, st);
}

template <typename Tin>
cudaError_t launch_pipe_d(const void *q, const void *k, const void *v, const float *g,
                          const float *beta, float *pool, const int32_t *slots, int num_slots,
                          void *out, int N, int H, int L, int dk, int dv, int *err, Prologue pro,
                          cudaStream_t st)
{
#define KDA_PIPE(DK_, DV_)                                                                          \
    if (dk == DK_ && dv == DV_)                                                                     \
        return launch_pipe_p<DK_, DV_, Tin>(q, k, v, g, beta, pool, slots, num_slots, out, N, H, L, \
                                            err, pro, st);
    KDA_PIPE(128, 128)
    KDA_PIPE(64, 64)
    KDA_PIPE(128, 64)
    KDA_PIPE(64, 128)
#undef KDA_PIPE
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_decode_pipe(const void *q, const void *k, const void *v, const float *g,
                               const float *beta, float *pool, const int32_t *slots, int num_slots,
                               void *out, int N, int H, int L, int dk, int dv, bool bf16, int *err,
                               Prologue pro, cudaStream_t st)
{
    if (N == 0 || L == 0) return cudaSuccess;
    // One token: nothing to overlap with the state stream, so the single-step
    // kernel (every load in flight at once) moves it faster; its per-token
    // arithmetic is the same operation for operation.
    if (L == 1)
        return launch_decode_slots(q, k, v, g, beta, pool, slots, num_slots, out, N, H, dk, dv,
                                   bf16, err, pro, st);
    if (bf16)
        return launch_pipe_d<__nv_bfloat16>(q, k, v, g, beta, pool, slots, num_slots, out, N, H, L,
                                            dk, dv, err, pro, st);
    return launch_pipe_d<float>(q, k, v, g, beta, pool, slots, num_slots, out, N, H, L, dk, dv, err,
                                pro, st);
}

}  // namespace kda

// chunk_prep.cu -- per-(chunk, head) intra-chunk work of the bf16 KDA prefill
// (dk = dv = 128, C = 64).  Fully parallel over (chunk, head); no state.
//
// Kimi Linear paper notes (paper-notes-site), section 3: inside a chunk the
// intra-chunk writes are gathered by a WY-like representation (W, U) and the
// output splits into an inter-chunk and an intra-chunk part; section 2 and
// the constrained-DPLR remark (with the Figure 2 note): KDA ties the low-rank
// factors to k, which saves matrix products and avoids the inverse
// cumulative-decay (1/Gamma) terms of the general DPLR form.  For one chunk of
// one head this kernel produces the record of chunk_ws.h:
//     G     = chunk-local inclusive cumsum of g          (per channel)
//     A_ij  = beta_i sum_c k_ic k_jc e^{G_ic - G_jc}     (j < i)
//     P_ij  =        sum_c q_ic k_jc e^{G_ic - G_jc}     (j <= i)
//     T     = (I + A)^-1                                  (unit lower-tri.)
//     W = T (beta K e^G),  U = T (beta V),  Qg = Q e^G,  Kt = K e^{G_C - G}
//
// Two ways to the same record, chosen per chunk inside one launch
// (chunk_prep_tc_kernel):
//
// 1. Chunk-start exponents on tcgen05 (the common case).  Every decayed form
//    is referenced at the chunk start: q e^G, beta k e^G, k e^{-G}.  Then A
//    and P are each one product of full tiles, and A/P, W and U are three
//    tcgen05 MMA groups with fp32 accumulators in tensor memory (see the
//    comment above chunk_prep_tc_kernel).  Valid while every e^{+-G} and
//    e^{G_C - G} of the chunk stays within e^{+-80}.
//
// 2. Sub-chunk exponents on mma.sync (prep_subchunk), for chunks outside that
//    range.  The chunk is cut into four sub-chunks of 16 tokens, I = 0..3,
//    with block-end cumsums R_I (R_{-1} = 0).  Per token and channel only
//    alpha = e^g is exponentiated; everything else is a product of alphas:
//        a_i = e^{G_i - R_{I-1}} (forward product within the block, <= 1)
//        b_i = e^{R_I - G_i}     (backward product within the block, <= 1)
//        d_I = e^{R_I - R_{I-1}} (block total)
//    For i in block I and j in block J:
//        J < I:  e^{G_i - G_j} = a_i * D_JI * b_j,  D_JI = prod_{J<M<I} d_M <= 1
//        J = I:  e^{G_i - G_j} = a_i * (1 / a_j),   1/a_j <= e^{16 * max|g|}
//    so with per-token g >= -5 no factor leaves e^{+-80}.
// Neither path forms a 1/Gamma over a span that could overflow.
//
// Both paths form T = (I + A)^-1 in fp32 (16x16 diagonal blocks by forward
// substitution, then the 2x2-block recursion T21 = -T22 A21 T11 at 16 and 32
// rows on tf32 tensor-core MMAs with fp32 accumulation) and round T once to
// bf16 for the W and U products.
#include <cudaTypedefs.h>

#include <mutex>

#include "chunk_ws.h"
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"
#include "prep_common.cuh"

namespace kda {
using namespace prep;
namespace {

constexpr int TILE = C * D * 2;   // bytes of a 64 x 128 bf16 tile

// 64 x 128 bf16 tile, 256-byte rows, 16-byte chunk j of row r at j ^ (r & 7)
__device__ __forceinline__ int toff(int r, int c) {
    return r * 256 + ((((c >> 3) ^ (r & 7))) << 4) + ((c & 7) << 1);
}
__device__ __forceinline__ int toff_chunk(int r, int j) {
    return r * 256 + (((j ^ (r & 7))) << 4);
}
// index of the (J, I) block pair, J < I
__device__ __forceinline__ int pair_idx(int J, int I) { return I * (I - 1) / 2 + J; }

struct __align__(16) PrepSmem {
    unsigned char Xq[TILE];   // q in; then q a          (then A, fp32 64x64)
    unsigned char Kb[TILE];   // k in; then k b
    unsigned char Vb[TILE];   // v in; then beta v
    unsigned char Xk[TILE];   // beta k a                (then T, fp32 64x64)
    unsigned char Kd[TILE];   // k / a                   (then T-recursion scratch)
    unsigned char KG[TILE];   // beta k e^G
    float Dm[6][D];           // D_JI per channel
    float d[4][D];            // block totals
    float beta[C];
    float rq[C], rk[C];       // prologue: per-row factors of q and k
};

__device__ __forceinline__ uint32_t scale_bf16x2(uint32_t x, float2 s) {
    __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162 *>(&x);
    return pack_bf16(__low2float(v) * s.x, __high2float(v) * s.y);
}

// A (isP = false: left operand beta k a) or P (isP = true: left operand q a)
// for row block Ib: 16 rows x 16 (Ib + 1) columns, on m16n8k16 bf16 MMAs.
// Ends with a CTA barrier (the operand tiles are then dead), after which A is
// written as fp32 over the Xq tile and P (masked, bf16) into the record.
template <int Ib>
__device__ __forceinline__ void ap_block(PrepSmem &sm, unsigned char *rec, bool isP, int lane) {
    const int gid = lane >> 2, tig = lane & 3;
    const unsigned char *X = isP ? sm.Xq : sm.Xk;
    float acc[Ib + 1][2][4];
#pragma unroll
    for (int J = 0; J <= Ib; ++J)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[J][nt][e] = 0.f;
    const int ar = 16 * Ib + (lane & 7) + 8 * ((lane >> 3) & 1);
    const int bn = (lane & 7) + 8 * (lane >> 4);
    const int bk = (lane >> 3) & 1;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
        uint32_t af[4];
        ldsm_x4(af, X + toff_chunk(ar, 2 * ks + (lane >> 4)));
#pragma unroll
        for (int J = 0; J <= Ib; ++J) {
            uint32_t bf[4];
            ldsm_x4(bf, (J < Ib ? sm.Kb : sm.Kd) + toff_chunk(16 * J + bn, 2 * ks + bk));
            if (J + 1 < Ib) {   // D_JI = 1 for adjacent blocks
                const float *dm = sm.Dm[pair_idx(J, Ib)];
                const float2 slo = *reinterpret_cast<const float2 *>(dm + 16 * ks + 2 * tig);
                const float2 shi = *reinterpret_cast<const float2 *>(dm + 16 * ks + 8 + 2 * tig);
                bf[0] = scale_bf16x2(bf[0], slo);
                bf[2] = scale_bf16x2(bf[2], slo);
                bf[1] = scale_bf16x2(bf[1], shi);
                bf[3] = scale_bf16x2(bf[3], shi);
            }
            mma_bf16(acc[J][0], af, bf[0], bf[1]);
            mma_bf16(acc[J][1], af, bf[2], bf[3]);
        }
    }
    __syncthreads();   // operand tiles are dead: Xq becomes A (fp32)
    float *Am = reinterpret_cast<float *>(sm.Xq);
#pragma unroll
    for (int J = 0; J < 4; ++J)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int i = 16 * Ib + gid + 8 * hh;
                const int j = 16 * J + 8 * nt + 2 * tig;
                float v0 = 0.f, v1 = 0.f;
                if (J <= Ib) { v0 = acc[J <= Ib ? J : 0][nt][2 * hh]; v1 = acc[J <= Ib ? J : 0][nt][2 * hh + 1]; }
                if (!isP) {
                    if (J <= Ib) {
                        Am[fsw(i, j)] = (j < i) ? v0 : 0.f;
                        Am[fsw(i, j + 1)] = (j + 1 < i) ? v1 : 0.f;
                    }
                } else {
                    v0 = (j <= i) ? v0 : 0.f;
                    v1 = (j + 1 <= i) ? v1 : 0.f;
                    *reinterpret_cast<uint32_t *>(rec + ws::OFF_P + ws::sw128(i, j)) = pack_bf16(v0, v1);
                }
            }
}

// T = (I + A)^-1 in fp32 for the strictly lower-triangular A (64 x 64, fsw
// layout): 16x16 diagonal blocks by forward substitution (warps 0-1, lane ->
// (block, column)), strictly-upper blocks zeroed (warps 2-7), then the 2x2-block
// recursion T21 = -T22 A21 T11 at 16 and 32 rows on tf32 tensor-core MMAs with
// fp32 accumulation.  Called by all 256 threads; ends with a CTA barrier.
__device__ __forceinline__ void form_T(const float *Am, float *Tm, float *Zs, int tid) {
    const int lane = tid & 31, warp = tid >> 5;
    const int gid = lane >> 2, tig = lane & 3;
    if (warp < 2) {
        // 16x16 diagonal blocks: lane -> (block, column)
        const int Bk = 2 * warp + (lane >> 4), c = lane & 15, o = 16 * Bk;
        float x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float s = 0.f;
#pragma unroll
            for (int j = 0; j < i; ++j) s += Am[fsw(o + i, o + j)] * x[j];
            x[i] = (i < c) ? 0.f : (i == c) ? 1.f : -s;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) Tm[fsw(o + i, o + c)] = x[i];
    } else {
        // zero the strictly-upper 16x16 blocks
        for (int e = tid - 64; e < 6 * 256; e += NT - 64) {
            const int blk = e >> 8, w = e & 255;
            const int Ib = blk < 3 ? 0 : blk < 5 ? 1 : 2;
            const int Jb = blk < 3 ? blk + 1 : blk < 5 ? blk - 1 : 3;
            Tm[fsw(16 * Ib + (w >> 4), 16 * Jb + (w & 15))] = 0.f;
        }
    }
    __syncthreads();
    // Off-diagonal blocks on the tensor cores (tf32, fp32 accumulate), one
    // 16x8 output tile per warp:
    //   16-row level: T_IJ = -T_II (A_IJ T_JJ) for (I, J) = (1, 0), (3, 2)
    //   32-row level: T[32:64, 0:32] = -T[32:64, 32:64] (A[32:64, 0:32] T[0:32, 0:32])
    // Zs holds the inner products at the coordinates of the block they feed.
    if (warp < 4) {
        const int Ib = (warp >> 1) ? 3 : 1, Jb = Ib - 1, n0 = 16 * Jb + 8 * (warp & 1);
        float c[4] = {0.f, 0.f, 0.f, 0.f};
        tile_tf32<16>(c, Am, 16 * Ib, 16 * Jb, Tm, 16 * Jb, n0, gid, tig);
        store_tile(Zs, c, 16 * Ib, n0, gid, tig, 1.f);
    }
    __syncthreads();
    if (warp < 4) {
        const int Ib = (warp >> 1) ? 3 : 1, Jb = Ib - 1, n0 = 16 * Jb + 8 * (warp & 1);
        float c[4] = {0.f, 0.f, 0.f, 0.f};
        tile_tf32<16>(c, Tm, 16 * Ib, 16 * Ib, Zs, 16 * Ib, n0, gid, tig);
        store_tile(Tm, c, 16 * Ib, n0, gid, tig, -1.f);
    }
    __syncthreads();
    {
        const int r0 = 32 + 16 * (warp >> 2), n0 = 8 * (warp & 3);
        float c[4] = {0.f, 0.f, 0.f, 0.f};
        tile_tf32<32>(c, Am, r0, 0, Tm, 0, n0, gid, tig);
        store_tile(Zs, c, r0, n0, gid, tig, 1.f);
        __syncthreads();
        float z[4] = {0.f, 0.f, 0.f, 0.f};
        tile_tf32<32>(z, Tm, r0, 32, Zs, 32, n0, gid, tig);
        store_tile(Tm, z, r0, n0, gid, tig, -1.f);
    }
    __syncthreads();
}

// Diagonal 16x16 blocks of A (fp32, fsw layout over Am) and of P (bf16, into
// the record) for a chunk whose decay inside a sub-chunk is so strong that
// the factorised form e^{G_i - G_j} = a_i (1 / a_j) leaves the fp32 range:
// every factor is formed directly as e^{G_i - G_j} = exp(sum of g over tokens
// j+1 .. i) <= 1 (for g <= 0), from q, k and g read again from global memory.
// Warp w takes the (block, column) tasks w, w + 8, ...; lane l the channels
// 4l .. 4l + 3.  Called by all 256 threads.
template <bool PRO>
__device__ __forceinline__ void ap_diag_direct(
    float *Am, unsigned char *rec, const float *sbeta, const float *srq, const float *srk,
    const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
    const float *__restrict__ g, size_t base, size_t row_stride, int len)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int c = 4 * lane;
    auto ld4 = [&](const __nv_bfloat16 *p, int r) {
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (r < len) {
            const uint2 w = *reinterpret_cast<const uint2 *>(p + base + (size_t)r * row_stride + c);
            const float2 lo = bf16x2_to_float2(w.x), hi = bf16x2_to_float2(w.y);
            x = make_float4(lo.x, lo.y, hi.x, hi.y);
        }
        return x;
    };
    for (int task = warp; task < 64; task += NT / 32) {
        const int I = task >> 4, jj = task & 15, j = 16 * I + jj;
        float4 kj = ld4(k, j);
        if (PRO) { const float f = srk[j]; kj.x *= f; kj.y *= f; kj.z *= f; kj.w *= f; }
        float4 sg = make_float4(0.f, 0.f, 0.f, 0.f);      // sum of g over tokens j+1 .. i
        for (int ii = jj; ii < 16; ++ii) {
            const int i = 16 * I + ii;
            if (ii > jj && i < len) {
                const float4 gi = *reinterpret_cast<const float4 *>(g + base + (size_t)i * row_stride + c);
                sg.x += gi.x; sg.y += gi.y; sg.z += gi.z; sg.w += gi.w;
            }
            float4 qi = ld4(q, i), ki = ld4(k, i);
            if (PRO) {
                const float fq = srq[i], fk = srk[i];
                qi.x *= fq; qi.y *= fq; qi.z *= fq; qi.w *= fq;
                ki.x *= fk; ki.y *= fk; ki.z *= fk; ki.w *= fk;
            }
            const float4 e = make_float4(expf(sg.x), expf(sg.y), expf(sg.z), expf(sg.w));
            const float4 ke = make_float4(kj.x * e.x, kj.y * e.y, kj.z * e.z, kj.w * e.w);
            float a = ki.x * ke.x + ki.y * ke.y + ki.z * ke.z + ki.w * ke.w;
            float pp = qi.x * ke.x + qi.y * ke.y + qi.z * ke.z + qi.w * ke.w;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                a += __shfl_xor_sync(0xffffffffu, a, o);
                pp += __shfl_xor_sync(0xffffffffu, pp, o);
            }
            if (lane == 0) {
                Am[fsw(i, j)] = ii > jj ? sbeta[i] * a : 0.f;
                *reinterpret_cast<__nv_bfloat16 *>(rec + ws::OFF_P + ws::sw128(i, j)) = __float2bfloat16_rn(pp);
            }
        }
    }
}

// The record of one (chunk, head) with every exponent referenced inside its
// 16-token sub-chunk.  The tensor-core prep below calls this for the chunks
// whose decay over the chunk leaves its exponent range.  Any g <= 0 is taken:
// when a sub-chunk's own decay underflows the factor a_j (1 / a_j would
// overflow), its diagonal blocks of A and P are formed directly
// (ap_diag_direct).  Called by all 256 threads of the CTA; smem_raw holds a PrepSmem.
template <bool PRO>
__device__ __noinline__ void prep_subchunk(
    unsigned char *smem_raw, const __nv_bfloat16 *__restrict__ q,
    const __nv_bfloat16 *__restrict__ k, const __nv_bfloat16 *__restrict__ v,
    const float *__restrict__ g, const float *__restrict__ beta, const int32_t *__restrict__ cu,
    const int32_t *__restrict__ coff, int N, int T, int total_T, int H, int cps,
    unsigned char *__restrict__ wsp, const Prologue &pro, int chunk, int h)
{
    PrepSmem &sm = *reinterpret_cast<PrepSmem *>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gid = lane >> 2, tig = lane & 3;

    int len;
    long long t0;
    locate_chunk(chunk, cu, coff, N, T, total_T, cps, t0, len);
    unsigned char *rec = wsp + ((size_t)chunk * H + h) * ws::RECORD;
    const size_t row_stride = (size_t)H * D;              // elements between tokens
    const size_t base = ((size_t)t0 * H + h) * D;         // element offset of (t0, h, 0)

    // ---- stage q, k, v (zero-filled past the end) ----
    {
        const uint32_t xq = smem_u32(sm.Xq), kb = smem_u32(sm.Kb), vb = smem_u32(sm.Vb);
#pragma unroll
        for (int it = 0; it < C * (D / 8) / NT; ++it) {
            const int i = tid + it * NT;
            const int r = i >> 4, j = i & 15;
            const bool ok = r < len;
            const size_t off = ok ? base + (size_t)r * row_stride + j * 8 : 0;
            const uint32_t so = toff_chunk(r, j), n = ok ? 16 : 0;
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(xq + so), "l"(q + off), "r"(n));
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(kb + so), "l"(k + off), "r"(n));
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(vb + so), "l"(v + off), "r"(n));
        }
    }
    cp_async_commit();

    // ---- elementwise ownership: sub-chunk I, channels c0, c0 + 1 ----
    const int I = tid >> 6, c0 = 2 * (tid & 63);
    float2 a[16], b[16];
    bool tiny_a;
    {
        float2 al[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int r = 16 * I + i;
            float2 gv = make_float2(0.f, 0.f);
            if (r < len) gv = *reinterpret_cast<const float2 *>(g + base + (size_t)r * row_stride + c0);
            al[i] = make_float2(expf(gv.x), expf(gv.y));
        }
        float2 run = make_float2(1.f, 1.f);
#pragma unroll
        for (int i = 0; i < 16; ++i) { run.x *= al[i].x; run.y *= al[i].y; a[i] = run; }
        tiny_a = !(run.x >= 0x1p-60f && run.y >= 0x1p-60f);   // a is smallest at the block end
        run = make_float2(1.f, 1.f);
#pragma unroll
        for (int i = 15; i >= 0; --i) { b[i] = run; run.x *= al[i].x; run.y *= al[i].y; }
    }
    sm.d[I][c0] = a[15].x;
    sm.d[I][c0 + 1] = a[15].y;
    if (tid < C) {
        float bt = (tid < len) ? beta[(size_t)(t0 + tid) * H + h] : 0.f;
        if (PRO && (pro.flags & kProBetaSigmoid) && tid < len) bt = sigmoid_f(bt);
        sm.beta[tid] = bt;
    }
    cp_async_wait<0>();
    __syncthreads();
    if (PRO) {
        // prologue: per-row factors (thread: tensor tid >> 7, row, half of the
        // row); rows past the end are zero and get factor 0
        const int tens = tid >> 7, rr = (tid >> 1) & 63, hf = tid & 1;
        float f = 1.f;
        if (pro.flags & kProQkL2Norm) {
            const unsigned char *tile = tens ? sm.Kb : sm.Xq;
            float ss = 0.f;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint4 x = *reinterpret_cast<const uint4 *>(tile + toff_chunk(rr, 8 * hf + j));
                const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const __nv_bfloat162 p2 = *reinterpret_cast<const __nv_bfloat162 *>(&w[e]);
                    const float a = __low2float(p2), b = __high2float(p2);
                    ss = fmaf(a, a, fmaf(b, b, ss));
                }
            }
            ss += __shfl_xor_sync(0xffffffffu, ss, 1);
            f = inv_norm(ss);
        }
        if (hf == 0) {
            if (tens) sm.rk[rr] = f;
            else sm.rq[rr] = f * pro.q_scale;
        }
        __syncthreads();
    }

    float2 E = make_float2(1.f, 1.f), F = make_float2(1.f, 1.f);
    {
        float2 dd[4];
#pragma unroll
        for (int J = 0; J < 4; ++J) dd[J] = make_float2(sm.d[J][c0], sm.d[J][c0 + 1]);
#pragma unroll
        for (int J = 0; J < 4; ++J) {
            if (J < I) { E.x *= dd[J].x; E.y *= dd[J].y; }
            if (J > I) { F.x *= dd[J].x; F.y *= dd[J].y; }
        }
        if (I == 0) {
            // e^{G_C} = product of all block totals
            float2 e = make_float2(dd[0].x * dd[1].x * dd[2].x * dd[3].x,
                                   dd[0].y * dd[1].y * dd[2].y * dd[3].y);
            *reinterpret_cast<float2 *>(rec + ws::OFF_EGC + c0 * 4) = e;
        }
        // D_JI for the pairs J < I of this thread's block I
#pragma unroll
        for (int J = 0; J < 3; ++J) {
            if (J < I) {
                float2 m = make_float2(1.f, 1.f);
#pragma unroll
                for (int M = 1; M < 3; ++M)
                    if (M > J && M < I) { m.x *= dd[M].x; m.y *= dd[M].y; }
                sm.Dm[pair_idx(J, I)][c0] = m.x;
                sm.Dm[pair_idx(J, I)][c0 + 1] = m.y;
            }
        }
    }
    {
        uint32_t kt[2][8];   // Kt for (channel, token pair) -> transposed store
        float2 kt_prev = make_float2(0.f, 0.f);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int r = 16 * I + i;
            const int o = toff(r, c0);
            const float br = sm.beta[r];
            const __nv_bfloat162 q2 = *reinterpret_cast<const __nv_bfloat162 *>(sm.Xq + o);
            const __nv_bfloat162 k2 = *reinterpret_cast<const __nv_bfloat162 *>(sm.Kb + o);
            const __nv_bfloat162 v2 = *reinterpret_cast<const __nv_bfloat162 *>(sm.Vb + o);
            float qx = __low2float(q2), qy = __high2float(q2);
            float kx = __low2float(k2), ky = __high2float(k2);
            const float vx = __low2float(v2), vy = __high2float(v2);
            if (PRO) {
                const float fq = sm.rq[r], fk = sm.rk[r];
                qx *= fq; qy *= fq; kx *= fk; ky *= fk;
            }
            const float2 ai = a[i], bi = b[i];
            *reinterpret_cast<uint32_t *>(sm.Xq + o) = pack_bf16(qx * ai.x, qy * ai.y);
            *reinterpret_cast<uint32_t *>(sm.Xk + o) = pack_bf16(br * kx * ai.x, br * ky * ai.y);
            *reinterpret_cast<uint32_t *>(sm.KG + o) =
                pack_bf16(br * kx * ai.x * E.x, br * ky * ai.y * E.y);
            *reinterpret_cast<uint32_t *>(sm.Kd + o) = pack_bf16(__fdividef(kx, ai.x), __fdividef(ky, ai.y));
            *reinterpret_cast<uint32_t *>(sm.Kb + o) = pack_bf16(kx * bi.x, ky * bi.y);
            *reinterpret_cast<uint32_t *>(sm.Vb + o) = pack_bf16(br * vx, br * vy);
            *reinterpret_cast<uint32_t *>(rec + ws::aw_off(64 + r, c0)) =
                pack_bf16(qx * ai.x * E.x, qy * ai.y * E.y);
            const float ktx = kx * bi.x * F.x, kty = ky * bi.y * F.y;
            if (i & 1) {
                kt[0][i >> 1] = pack_bf16(kt_prev.x, ktx);
                kt[1][i >> 1] = pack_bf16(kt_prev.y, kty);
            } else {
                kt_prev = make_float2(ktx, kty);
            }
        }
#pragma unroll
        for (int e = 0; e < 2; ++e)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int c = c0 + e;
                *reinterpret_cast<uint4 *>(rec + ws::OFF_KTT + ws::sw128(c, 16 * I + 8 * hh)) =
                    make_uint4(kt[e][4 * hh], kt[e][4 * hh + 1], kt[e][4 * hh + 2], kt[e][4 * hh + 3]);
            }
    }
    __syncthreads();

    // ---- A (warps 0-3) and P (warps 4-7) for row block Ib = warp & 3 ----
    switch (warp & 3) {
        case 0: ap_block<0>(sm, rec, warp >= 4, lane); break;
        case 1: ap_block<1>(sm, rec, warp >= 4, lane); break;
        case 2: ap_block<2>(sm, rec, warp >= 4, lane); break;
        default: ap_block<3>(sm, rec, warp >= 4, lane); break;
    }
    // a sub-chunk decay below 2^-60 makes 1 / a_j unusable: diagonal blocks directly
    if (__syncthreads_or(tiny_a)) {
        ap_diag_direct<PRO>(reinterpret_cast<float *>(sm.Xq), rec, sm.beta, sm.rq, sm.rk, q, k, g,
                            base, row_stride, len);
        __syncthreads();
    }

    // ---- T = (I + A)^-1 in fp32 ----
    const float *Am = reinterpret_cast<const float *>(sm.Xq);
    float *Tm = reinterpret_cast<float *>(sm.Xk);
    form_T(Am, Tm, reinterpret_cast<float *>(sm.Kd), tid);

    // ---- W = T (beta K e^G) (warps 0-3), U = T (beta V) (warps 4-7) ----
    {
        const bool isU = warp >= 4;
        const int qd = warp & 3;                       // 32-channel quarter
        const unsigned char *Bs = isU ? sm.Vb : sm.KG;
        float acc[4][4][4];
#pragma unroll
        for (int Ib = 0; Ib < 4; ++Ib)
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[Ib][nt][e] = 0.f;
        const int bkr = (lane & 7) + 8 * ((lane >> 3) & 1);
#pragma unroll
        for (int Ib = 0; Ib < 4; ++Ib)
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                if (ks <= Ib) {
                    const int r0 = 16 * Ib + gid, k0 = 16 * ks + 2 * tig;
                    uint32_t af[4];
                    const float2 t00 = *reinterpret_cast<const float2 *>(&Tm[fsw(r0, k0)]);
                    const float2 t10 = *reinterpret_cast<const float2 *>(&Tm[fsw(r0 + 8, k0)]);
                    const float2 t01 = *reinterpret_cast<const float2 *>(&Tm[fsw(r0, k0 + 8)]);
                    const float2 t11 = *reinterpret_cast<const float2 *>(&Tm[fsw(r0 + 8, k0 + 8)]);
                    af[0] = pack_bf16(t00.x, t00.y);
                    af[1] = pack_bf16(t10.x, t10.y);
                    af[2] = pack_bf16(t01.x, t01.y);
                    af[3] = pack_bf16(t11.x, t11.y);
#pragma unroll
                    for (int np = 0; np < 2; ++np) {
                        uint32_t bf[4];
                        const int kr = 16 * ks + bkr;
                        ldsm_x4_t(bf, Bs + toff_chunk(kr, 4 * qd + 2 * np + (lane >> 4)));
                        mma_bf16(acc[Ib][2 * np], af, bf[0], bf[1]);
                        mma_bf16(acc[Ib][2 * np + 1], af, bf[2], bf[3]);
                    }
                }
            }
#pragma unroll
        for (int Ib = 0; Ib < 4; ++Ib)
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int r = 16 * Ib + gid + 8 * hh;
                    const int n = 32 * qd + 8 * nt + 2 * tig;
                    const uint32_t pk = pack_bf16(acc[Ib][nt][2 * hh], acc[Ib][nt][2 * hh + 1]);
                    if (isU)
                        *reinterpret_cast<uint32_t *>(rec + ws::OFF_U + (size_t)qd * ws::U_TILE + r * 64 +
                                                      ((n & 31) << 1)) = pk;
                    else
                        *reinterpret_cast<uint32_t *>(rec + ws::aw_off(r, n)) = pk;
                }
    }
}

// ---------------------------------------------------------------------------
// Tensor-core prep: the same record, every exponent referenced at the chunk
// start.  With G the chunk-local inclusive cumsum,
//     A_ij = (beta_i k_i e^{G_i}) . (k_j e^{-G_j})   (j < i)
//     P_ij = (q_i e^{G_i}) . (k_j e^{-G_j})          (j <= i)
// exactly; the factors are formed once per token and channel, so A and P are
// each one product of full tiles.  This is used when every e^{+-G_i} and
// e^{G_C - G_i} of the chunk lies within e^{+-80} (normal fp32 and bf16
// numbers; for g <= 0 that is G_C >= -80, an average per-token g >= -1.25).
// A chunk outside that range is done by prep_subchunk in the same CTA.
//
// Inputs arrive by TMA (tensor maps over [tokens, heads, channels]; no
// multicast), which keeps ~80 KB per CTA in flight where per-thread copies
// were limited to ~20 GB/s per SM.  Products on tcgen05 (one issuing thread,
// fp32 accumulators in TMEM):
//   MMA-AP  [beta K e^G ; Q e^G] (128 x 128) x (K e^{-G})^T  -> TMEM cols 0-63
//           (lanes 0-63: A before masking, lanes 64-127: P before masking)
//   MMA-W   [T ; *] (128 x 64) x beta K e^G (64 x 128)        -> cols 0-127, lanes 0-63
//   MMA-U   [* ; T] (128 x 64) x beta V     (64 x 128)        -> cols 128-255, lanes 64-127
// The rows marked * are whatever lies next to T in shared memory; their
// products land in TMEM lanes that are never read.  T itself comes from
// form_T_padded_diag (fp32).  K^T leaves from the registers of the forms
// pass; q e^G and P by bulk async stores of their shared-memory images; W
// and U, the last, by a coalesced copy of all threads so that the CTA need
// not wait for a bulk copy to read them.
// ---------------------------------------------------------------------------
namespace tcp {
// Tiles are K-major with the 128-byte swizzle (rows of 64 bf16 = 128 bytes,
// 16-byte chunk j of row r at j ^ (r % 8), 8-row groups 1024 bytes apart), as
// TMA writes them with SWIZZLE_128B.  Read with rows = tokens they are the
// K-major A operands of MMA-AP; the same bytes are the MN-major B operands of
// MMA-W and MMA-U (tokens along K, 64-channel atoms along N).
constexpr int OFF_KQ = 0;              // per 64-channel block b at b * 16384:
                                       //   [k -> beta k e^G : 64 rows][q -> q e^G : 64 rows]
constexpr int OFF_KI = 32768;          // k e^{-G} (block b at b * 8192); then A (fp32 64 x 64)
constexpr int OFF_Z = 49152;           // the padded diagonal blocks of A; then form_T scratch
constexpr int OFF_G = OFF_KI;          // g (fp32 [64][128], TMA) until the cumsum has read it
constexpr int OFF_V = 65536;           // v -> beta v (block b at b * 8192)
constexpr int OFF_TB = 81920;          // P image, then T (bf16, 64 swizzled rows)
constexpr int OFF_TM = 90112;          // T (fp32 64 x 64); also the rows after T in MMA-W's A
constexpr int OFF_GS = 106496;         // per-sub-chunk sums of g [4][128]
constexpr int OFF_BETA = OFF_GS + 4 * D * 4;
constexpr int OFF_RQ = OFF_BETA + C * 4;
constexpr int OFF_RK = OFF_RQ + C * 4;
constexpr int END = OFF_RK + C * 4;
// mbarriers and the TMEM slot sit past both this layout and PrepSmem, so the
// fallback never overwrites them
constexpr int OFF_BAR = (int)((((size_t)END > sizeof(PrepSmem) ? (size_t)END : sizeof(PrepSmem)) + 15) & ~(size_t)15);
constexpr int BYTES = OFF_BAR + 32;
constexpr uint32_t TX_QKV = 6 * 8192;          // q, k, v: two 64-channel boxes each
constexpr uint32_t TX_G = C * D * 4;            // g
constexpr uint32_t TMEM_COLS = 256;
constexpr float RANGE2 = 80.f * 1.4426950408889634f;   // e^{+-80} bound, in log2 units
// byte offset of (row r, channel c in 0..63) in a swizzled 64-channel block
__device__ __forceinline__ int sw(int r, int c) {
    return r * 128 + ((((c >> 3) ^ (r & 7))) << 4) + ((c & 7) << 1);
}
}  // namespace tcp

template <bool PRO>
__global__ void __launch_bounds__(NT, 2)
chunk_prep_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                     const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                     const __nv_bfloat16 *__restrict__ v, const float *__restrict__ g,
                     const float *__restrict__ beta, const int32_t *__restrict__ cu,
                     const int32_t *__restrict__ coff, int N, int T, int total_T, int H, int cps,
                     unsigned char *__restrict__ wsp, Prologue pro, int *__restrict__ err)
{
    using namespace sm100;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // heads fastest and chunks last-to-first: the records written last, still
    // in L2 when the chain starts, are the first chunks of every head, the
    // ones the chain reads first
    const int lin = blockIdx.y * gridDim.x + blockIdx.x;
    const int h = lin % H, chunk = gridDim.x - 1 - lin / H;
    if (cu && chunk >= coff[N]) return;

    int len;
    long long t0;
    locate_chunk(chunk, cu, coff, N, T, total_T, cps, t0, len);
    unsigned char *rec = wsp + ((size_t)chunk * H + h) * ws::RECORD;
    uint64_t *bar_ld = reinterpret_cast<uint64_t *>(sm + tcp::OFF_BAR);
    uint64_t *bar = bar_ld + 1;
    uint64_t *bar_g = bar_ld + 3;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + tcp::OFF_BAR + 16);
    float *gs = reinterpret_cast<float *>(sm + tcp::OFF_GS);
    float *bet = reinterpret_cast<float *>(sm + tcp::OFF_BETA);
    float *rq = reinterpret_cast<float *>(sm + tcp::OFF_RQ);
    float *rk = reinterpret_cast<float *>(sm + tcp::OFF_RK);

    // ---- stage q, k, v (two 64-channel boxes each) and g by TMA; rows past
    // the sequence end are masked below, rows past the tensor read as zero ----
    if (tid == 0) {
        mbar_init(bar_ld, 1);
        mbar_init(bar, 1);
        mbar_init(bar_g, 1);
        fence_mbar_init();
        // g first, on its own barrier: the cumsum and the range check run
        // while q, k and v are still arriving
        mbar_arrive_expect_tx(bar_g, tcp::TX_G);
        const int tt = (int)t0;
        tma_load_3d(sm + tcp::OFF_G, &tm_g, 0, h, tt, bar_g);
        mbar_arrive_expect_tx(bar_ld, tcp::TX_QKV);
#pragma unroll
        for (int b = 0; b < 2; ++b) {
            tma_load_3d(sm + tcp::OFF_KQ + b * 16384, &tm_k, 64 * b, h, tt, bar_ld);
            tma_load_3d(sm + tcp::OFF_KQ + b * 16384 + 8192, &tm_q, 64 * b, h, tt, bar_ld);
            tma_load_3d(sm + tcp::OFF_V + b * 8192, &tm_v, 64 * b, h, tt, bar_ld);
        }
    }
    if (tid < C) {
        float bt = (tid < len) ? beta[(size_t)(t0 + tid) * H + h] : 0.f;
        if (PRO && (pro.flags & kProBetaSigmoid) && tid < len) bt = sigmoid_f(bt);
        bet[tid] = bt;
    }
    if (warp == 0) { tmem_alloc(tslot, tcp::TMEM_COLS); tmem_relinquish(); }
    bool ok = true;
    if (tid == 0) ok = mbar_wait(bar_g, 0);
    tc_fence_before();
    ok = __syncthreads_and(ok);
    tc_fence_after();
    const uint32_t tmem = *tslot;

    // ---- g: thread (sub-chunk I, channels c0, c0 + 1); local cumsum ----
    const int I = tid >> 6, c0 = 2 * (tid & 63);
    const int cb = c0 >> 6, cc = c0 & 63;          // 64-channel block, channel within it
    float2 G[16];
    {
        const float *gsm = reinterpret_cast<const float *>(sm + tcp::OFF_G);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int r = 16 * I + i;
            G[i] = make_float2(0.f, 0.f);
            if (r < len) G[i] = *reinterpret_cast<const float2 *>(gsm + r * D + c0);
        }
    }
    // cumsum in log2 units (G log2(e)), so that every e^{...} below is one ex2
    constexpr float L2E = 1.4426950408889634f;
    G[0].x *= L2E; G[0].y *= L2E;
#pragma unroll
    for (int i = 1; i < 16; ++i) { G[i].x = fmaf(G[i].x, L2E, G[i - 1].x); G[i].y = fmaf(G[i].y, L2E, G[i - 1].y); }
    *reinterpret_cast<float2 *>(gs + I * D + c0) = G[15];
    __syncthreads();

    // ---- prefix of the earlier sub-chunks; chunk total G_C; range check ----
    float2 GC = make_float2(0.f, 0.f), PF = make_float2(0.f, 0.f);
#pragma unroll
    for (int J = 0; J < 4; ++J) {
        const float2 sj = *reinterpret_cast<const float2 *>(gs + J * D + c0);
        if (J < I) { PF.x += sj.x; PF.y += sj.y; }
        GC.x += sj.x; GC.y += sj.y;
    }
    bool bad = !ok;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        G[i].x += PF.x; G[i].y += PF.y;
        bad |= !(fabsf(G[i].x) <= tcp::RANGE2 && fabsf(G[i].y) <= tcp::RANGE2 &&
                 GC.x - G[i].x <= tcp::RANGE2 && GC.y - G[i].y <= tcp::RANGE2);
    }
    // q, k, v have landed before anything (this path or the fallback, which
    // reuses the shared memory) touches their tiles
    if (tid == 0 && ok) ok = mbar_wait(bar_ld, 0);
    ok = __syncthreads_and(ok);
    if (__syncthreads_or(bad || !ok)) {
        // out of the chunk-start range (or a staging wait ran out): 16-token
        // references, mma.sync products, its own loads
        if (!ok && tid == 0) set_device_error(err, kErrWaitTimeout);
        if (ok) prep_subchunk<PRO>(sm, q, k, v, g, beta, cu, coff, N, T, total_T, H, cps, wsp, pro, chunk, h);
        __syncthreads();
        if (warp == 0) tmem_dealloc(tmem, tcp::TMEM_COLS);
        return;
    }

    if (PRO) {
        // per-row factors (thread: tensor tid >> 7, row, 64-channel block)
        const int tens = tid >> 7, rr = (tid >> 1) & 63, hf = tid & 1;
        float f = 1.f;
        if (pro.flags & kProQkL2Norm) {
            const unsigned char *row = sm + tcp::OFF_KQ + hf * 16384 + (tens ? 0 : 8192) + rr * 128;
            float ss = 0.f;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint4 x = *reinterpret_cast<const uint4 *>(row + 16 * j);
                const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 p2 = bf16x2_to_float2(w[e]);
                    ss = fmaf(p2.x, p2.x, fmaf(p2.y, p2.y, ss));
                }
            }
            ss += __shfl_xor_sync(0xffffffffu, ss, 1);
            f = inv_norm(ss);
        }
        if (hf == 0) {
            if (tens) rk[rr] = f;
            else rq[rr] = f * pro.q_scale;
        }
        __syncthreads();
    }

    // ---- decayed forms: q e^G, beta k e^G, beta v (in place), k e^{-G}
    // (over the consumed g), K e^{G_C - G} image, q e^G and e^{G_C} (record) ----
    {
        const float2 egc = make_float2(ex2_approx(GC.x), ex2_approx(GC.y));
        if (I == 0) *reinterpret_cast<float2 *>(rec + ws::OFF_EGC + c0 * 4) = make_float2(exp2f(GC.x), exp2f(GC.y));
        uint32_t kt[2][8];
        float2 kt_prev = make_float2(0.f, 0.f);
        unsigned char *kq = sm + tcp::OFF_KQ + cb * 16384;
        unsigned char *ki = sm + tcp::OFF_KI + cb * 8192;
        unsigned char *vv = sm + tcp::OFF_V + cb * 8192;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int r = 16 * I + i;
            const int o = tcp::sw(r, cc);
            const float2 eg = make_float2(ex2_approx(G[i].x), ex2_approx(G[i].y));
            const float2 em = make_float2(ex2_approx(-G[i].x), ex2_approx(-G[i].y));
            float2 qf = bf16x2_to_float2(*reinterpret_cast<const uint32_t *>(kq + 8192 + o));
            float2 kf = bf16x2_to_float2(*reinterpret_cast<const uint32_t *>(kq + o));
            float2 vf = bf16x2_to_float2(*reinterpret_cast<const uint32_t *>(vv + o));
            if (r >= len) { qf = kf = vf = make_float2(0.f, 0.f); }
            if (PRO) {
                const float fq = rq[r], fk = rk[r];
                qf = __fmul2_rn(qf, make_float2(fq, fq));
                kf = __fmul2_rn(kf, make_float2(fk, fk));
            }
            const float br = bet[r];
            const float2 b2 = make_float2(br, br);
            const uint32_t qg = pack_bf16x2(__fmul2_rn(qf, eg));
            const float2 kinv = __fmul2_rn(kf, em);
            const float2 kt2 = __fmul2_rn(kinv, egc);
            *reinterpret_cast<uint32_t *>(kq + 8192 + o) = qg;
            *reinterpret_cast<uint32_t *>(kq + o) = pack_bf16x2(__fmul2_rn(__fmul2_rn(kf, b2), eg));
            *reinterpret_cast<uint32_t *>(ki + o) = pack_bf16x2(kinv);
            *reinterpret_cast<uint32_t *>(vv + o) = pack_bf16x2(__fmul2_rn(vf, b2));
            if (i & 1) {
                kt[0][i >> 1] = pack_bf16(kt_prev.x, kt2.x);
                kt[1][i >> 1] = pack_bf16(kt_prev.y, kt2.y);
            } else {
                kt_prev = kt2;
            }
        }
        // K e^{G_C - G} transposed (channel rows, 64 tokens, 128-byte swizzle)
        // straight into the record: tokens 16 I .. 16 I + 15 of a row are the
        // 16-byte chunks 2I and 2I + 1, which the swizzle (XOR with row & 7)
        // keeps in one aligned 32-byte pair, swapped when row & 7 is odd: one
        // 256-bit store per row
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int r = c0 + e, x = r & 7;
            unsigned char *dst = rec + ws::OFF_KTT + r * 128 + ((((2 * I) ^ x) & ~1) << 4);
            const bool sw = x & 1;
            asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};\n" ::"l"(dst),
                         "r"(sw ? kt[e][4] : kt[e][0]), "r"(sw ? kt[e][5] : kt[e][1]), "r"(sw ? kt[e][6] : kt[e][2]),
                         "r"(sw ? kt[e][7] : kt[e][3]), "r"(sw ? kt[e][0] : kt[e][4]), "r"(sw ? kt[e][1] : kt[e][5]),
                         "r"(sw ? kt[e][2] : kt[e][6]), "r"(sw ? kt[e][3] : kt[e][7])
                         : "memory");
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();

    const uint32_t sb = smem_u32(sm);
    if (tid == 0) {
        tc_fence_after();
        // A: [beta k e^G ; q e^G] K-major (M = 128), B: k e^{-G} K-major (N = 64)
        constexpr uint32_t ID_AP = idesc_bf16(128, 64, false);
        const DescParts da = smem_desc_parts(sb + tcp::OFF_KQ, 16, 1024, 2);
        const DescParts db = smem_desc_parts(sb + tcp::OFF_KI, 16, 1024, 2);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
            umma_bf16_p(tmem, da.lo + (((kk >> 2) * 16384 + (kk & 3) * 32) >> 4), da.hi,
                        db.lo + (((kk >> 2) * 8192 + (kk & 3) * 32) >> 4), db.hi, ID_AP, kk > 0);
        umma_commit(bar);
        // the record part that is final now: q e^G (the swizzled q e^G tile
        // is already the record's layout for rows 64-127; nothing overwrites
        // it before form_T waits for the reads)
        bulk_s2g(rec + ws::OFF_AW + 8192, sm + tcp::OFF_KQ + 8192, 8192);
        bulk_s2g(rec + ws::OFF_AW + 16384 + 8192, sm + tcp::OFF_KQ + 16384 + 8192, 8192);
        bulk_commit();
    }
    // one thread waits for the MMA; the others sleep at the barrier
    if (tid == 0) ok = mbar_wait(bar, 0);
    ok = __syncthreads_and(ok);
    tc_fence_after();

    // ---- A (masked j < i) -> fp32 for form_T; P (masked j <= i) -> record ----
    float *Am = reinterpret_cast<float *>(sm + tcp::OFF_KI);
    float *Tm = reinterpret_cast<float *>(sm + tcp::OFF_TM);
    float *Ad = reinterpret_cast<float *>(sm + tcp::OFF_Z);
    if (ok && warp < 4) {
        float x[64];
        const uint32_t ta = tmem + ((uint32_t)(warp * 32) << 16);
        tmem_ld32(ta, *reinterpret_cast<float (*)[32]>(&x[0]));
        tmem_ld32(ta + 32, *reinterpret_cast<float (*)[32]>(&x[32]));
        tmem_wait_ld();
        const int i = (warp & 1) * 32 + lane;
        if (warp < 2) {
#pragma unroll
            for (int j4 = 0; j4 < 16; ++j4) {
                float4 a4;
                a4.x = (4 * j4 < i) ? x[4 * j4] : 0.f;
                a4.y = (4 * j4 + 1 < i) ? x[4 * j4 + 1] : 0.f;
                a4.z = (4 * j4 + 2 < i) ? x[4 * j4 + 2] : 0.f;
                a4.w = (4 * j4 + 3 < i) ? x[4 * j4 + 3] : 0.f;
                *reinterpret_cast<float4 *>(Am + i * 64 + 4 * (j4 ^ (i & 7))) = a4;
            }
            // the row's diagonal block, padded copy for the substitution: warp
            // w holds rows 32w..32w+31, i.e. diagonal blocks 2w (lanes 0-15)
            // and 2w + 1 (lanes 16-31)
            float *adr = Ad + (i >> 4) * (16 * 17) + (i & 15) * 17;
            const int ii = i & 15;
            const bool upper = lane >= 16;
            if (warp == 0) {
#pragma unroll
                for (int jj = 0; jj < 16; ++jj) adr[jj] = (jj < ii) ? (upper ? x[16 + jj] : x[jj]) : 0.f;
            } else {
#pragma unroll
                for (int jj = 0; jj < 16; ++jj) adr[jj] = (jj < ii) ? (upper ? x[48 + jj] : x[32 + jj]) : 0.f;
            }
        } else {
            unsigned char *img = sm + tcp::OFF_TB;
#pragma unroll
            for (int jc = 0; jc < 8; ++jc) {
                uint32_t pk[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int j = 8 * jc + 2 * e;
                    pk[e] = pack_bf16(j <= i ? x[j] : 0.f, j + 1 <= i ? x[j + 1] : 0.f);
                }
                *reinterpret_cast<uint4 *>(img + i * 128 + ((jc ^ (i & 7)) << 4)) =
                    make_uint4(pk[0], pk[1], pk[2], pk[3]);
            }
            fence_proxy_async_smem();
        }
    }
    tc_fence_before();
    __syncthreads();
    if (ok) {
        if (tid == 0) {
            bulk_s2g(rec + ws::OFF_P, sm + tcp::OFF_TB, 8192);
            bulk_commit();
        }
        form_T_padded_diag(Am, Ad, Tm, reinterpret_cast<float *>(sm + tcp::OFF_Z), tid);
        // T -> bf16, one swizzled 128-byte row per token row i
        {
            const int i = tid >> 2, jq = tid & 3;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int jg = 2 * jq + hh;
                const float4 lo = *reinterpret_cast<const float4 *>(Tm + i * 64 + 4 * ((2 * jg) ^ (i & 7)));
                const float4 hi = *reinterpret_cast<const float4 *>(Tm + i * 64 + 4 * ((2 * jg + 1) ^ (i & 7)));
                *reinterpret_cast<uint4 *>(sm + tcp::OFF_TB + i * 128 + ((jg ^ (i & 7)) << 4)) =
                    make_uint4(pack_bf16(lo.x, lo.y), pack_bf16(lo.z, lo.w), pack_bf16(hi.x, hi.y),
                               pack_bf16(hi.z, hi.w));
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            // A: [T ; *] and [* ; T] K-major (K = 64 tokens in one swizzled row);
            // B: beta k e^G and beta v as MN-major operands (tokens along K,
            // 64-channel atoms along N: LBO = atom stride, SBO = 8-token group)
            constexpr uint32_t ID_WU = idesc_bf16(128, 128, true);
            const DescParts ta = smem_desc_parts(sb + tcp::OFF_TB, 16, 1024, 2);
            const DescParts tu = smem_desc_parts(sb + tcp::OFF_TB - 8192, 16, 1024, 2);
            const DescParts bw = smem_desc_parts(sb + tcp::OFF_KQ, 16384, 1024, 2);
            const DescParts bu = smem_desc_parts(sb + tcp::OFF_V, 8192, 1024, 2);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                umma_bf16_p(tmem, ta.lo + ((kk * 32) >> 4), ta.hi, bw.lo + ((kk * 2048) >> 4), bw.hi, ID_WU, kk > 0);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                umma_bf16_p(tmem + 128, tu.lo + ((kk * 32) >> 4), tu.hi, bu.lo + ((kk * 2048) >> 4), bu.hi, ID_WU,
                            kk > 0);
            umma_commit(bar);
        }
        if (tid == 0) ok = mbar_wait(bar, 1);
        ok = __syncthreads_and(ok);
        tc_fence_after();
        if (ok) {
            // W rows (TMEM lanes 0-63, cols 0-127) and U rows (lanes 64-127,
            // cols 128-255); warp w: lane quarter w & 3, column half w >> 2
            const int qd = warp & 3, hf = warp >> 2;
            const int r = (qd & 1) * 32 + lane;
            float x[64];
            const uint32_t ta = tmem + ((uint32_t)(qd * 32) << 16) + (qd < 2 ? 0u : 128u) + 64u * hf;
            tmem_ld32(ta, *reinterpret_cast<float (*)[32]>(&x[0]));
            tmem_ld32(ta + 32, *reinterpret_cast<float (*)[32]>(&x[32]));
            tmem_wait_ld();
            // record images: W block hf (rows 0-63 of [W; Qg]) over the dead k
            // rows of block hf, U (four 64 x 32 tiles) over the dead v tile;
            // copied out below by all threads
            if (qd < 2) {
                unsigned char *dst = sm + tcp::OFF_KQ + hf * 16384 + r * 128;
#pragma unroll
                for (int jc = 0; jc < 8; ++jc)
                    *reinterpret_cast<uint4 *>(dst + ((jc ^ (r & 7)) << 4)) =
                        make_uint4(pack_bf16(x[8 * jc], x[8 * jc + 1]), pack_bf16(x[8 * jc + 2], x[8 * jc + 3]),
                                   pack_bf16(x[8 * jc + 4], x[8 * jc + 5]), pack_bf16(x[8 * jc + 6], x[8 * jc + 7]));
            } else {
#pragma unroll
                for (int tt = 0; tt < 2; ++tt) {
                    unsigned char *dst = sm + tcp::OFF_V + (2 * hf + tt) * ws::U_TILE + r * 64;
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float *xs = x + 32 * tt + 8 * e;
                        *reinterpret_cast<uint4 *>(dst + 16 * e) =
                            make_uint4(pack_bf16(xs[0], xs[1]), pack_bf16(xs[2], xs[3]),
                                       pack_bf16(xs[4], xs[5]), pack_bf16(xs[6], xs[7]));
                    }
                }
            }
        }
        __syncthreads();
        if (ok) {
            // all threads copy the 32 KB of images out with coalesced 16-byte
            // accesses (W block 0, W block 1, the four U tiles); nothing is
            // left in flight that reads shared memory
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int c = tid + NT * j;                   // 16-byte chunk, 0..2047
                const int src = c < 512 ? tcp::OFF_KQ + 16 * c
                              : c < 1024 ? tcp::OFF_KQ + 16384 + 16 * (c - 512) : tcp::OFF_V + 16 * (c - 1024);
                const size_t dst = c < 512 ? ws::OFF_AW + 16 * c
                                 : c < 1024 ? ws::OFF_AW + 16384 + 16 * (c - 512) : ws::OFF_U + 16 * (c - 1024);
                *reinterpret_cast<uint4 *>(rec + dst) = *reinterpret_cast<const uint4 *>(sm + src);
            }
        }
    }
    // the shared-memory sources of the bulk stores must be read before exit
    if (tid == 0) bulk_wait_read();
    if (!ok && tid == 0) set_device_error(err, kErrWaitTimeout);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, tcp::TMEM_COLS);
}

// Chunk offsets per sequence for varlen mode: coff[n] = sum_{m<n} ceil(len_m / C).
__global__ void chunk_plan_kernel(const int32_t *__restrict__ cu, int N, int total_T,
                                  int32_t *__restrict__ coff, int32_t *__restrict__ order)
{
    __shared__ int part[1024];
    const int tid = threadIdx.x;
    const int per = (N + 1023) / 1024;
    const int s0 = tid * per, s1 = min(N, s0 + per);
    int sum = 0;
    for (int n = s0; n < s1; ++n) {
        const int b = min(max(cu[n], 0), total_T), e = min(max(cu[n + 1], 0), total_T);
        sum += e > b ? (e - b + C - 1) / C : 0;
    }
    part[tid] = sum;
    __syncthreads();
    for (int off = 1; off < 1024; off <<= 1) {
        const int x = tid >= off ? part[tid - off] : 0;
        __syncthreads();
        part[tid] += x;
        __syncthreads();
    }
    int run = tid > 0 ? part[tid - 1] : 0;
    for (int n = s0; n < s1; ++n) {
        coff[n] = run;
        const int b = min(max(cu[n], 0), total_T), e = min(max(cu[n + 1], 0), total_T);
        run += e > b ? (e - b + C - 1) / C : 0;
    }
    if (tid == 1023) coff[N] = part[1023];
    if (order) {
        // rank of each sequence by decreasing length, ties by index (a
        // permutation); quadratic, so only for up to 4096 sequences
        for (int n = tid; n < N; n += 1024) {
            int rank = n;
            if (N <= 4096) {
                auto len = [&](int m) {
                    const int b = min(max(cu[m], 0), total_T), e = min(max(cu[m + 1], 0), total_T);
                    return e > b ? e - b : 0;
                };
                const int ln = len(n);
                rank = 0;
                for (int m = 0; m < N; ++m) {
                    const int lm = len(m);
                    rank += (lm > ln || (lm == ln && m < n)) ? 1 : 0;
                }
            }
            order[rank] = n;
        }
    }
}

}  // namespace

size_t chunk_prep_smem_bytes() { return tcp::BYTES + 1024; }

cudaError_t launch_chunk_plan(const int32_t *cu, int N, int total_T, int32_t *coff,
                              cudaStream_t st, int32_t *order)
{
    chunk_plan_kernel<<<1, 1024, 0, st>>>(cu, N, total_T, coff, order);
    return cudaGetLastError();
}

cudaError_t launch_chunk_prep(const void *q, const void *k, const void *v, const float *g,
                              const float *beta, const int32_t *cu, const int32_t *coff,
                              int N, int T, int total_T, int H, int max_chunks,
                              unsigned char *wsp, Prologue pro, int *err, cudaStream_t st)
{
    CUtensorMap mq, mk, mv, mg;
    cudaError_t e = make_token_map(&mq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, H, total_T, 64,
                                   CU_TENSOR_MAP_SWIZZLE_128B);
    if (e == cudaSuccess)
        e = make_token_map(&mk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, H, total_T, 64, CU_TENSOR_MAP_SWIZZLE_128B);
    if (e == cudaSuccess)
        e = make_token_map(&mv, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, H, total_T, 64, CU_TENSOR_MAP_SWIZZLE_128B);
    if (e == cudaSuccess)
        e = make_token_map(&mg, g, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, H, total_T, D, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (e != cudaSuccess) return e;
    const size_t smem = tcp::BYTES + 1024;
    const bool use_pro = pro.flags != 0 || pro.q_scale != 1.f;
    auto kern = use_pro ? chunk_prep_tc_kernel<true> : chunk_prep_tc_kernel<false>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int cps = (T + C - 1) / C;
    dim3 grid(max_chunks, H);
    kern<<<grid, NT, smem, st>>>(
        mq, mk, mv, mg, (const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)v, g,
        beta, cu, coff, N, T, total_T, H, cps, wsp, pro, err);
    return cudaGetLastError();
}

}  // namespace kda

// recurrent_bwd.cu -- gradients of the KDA recurrence (training backward),
// one warp per (sequence, head, 4-column tile of the state), eight warps
// (32 columns) per CTA.
//
// Kimi Linear paper notes (paper-notes-site), section 2: per token
//     S' = Diag(a) S_{t-1},  a = exp(g);  w = S'^T k;  u = beta (v - w);
//     S_t = S' + k u^T;  o_t = S_t^T q.
// The chain rule, token by token in reverse, with dS the gradient of the
// loss with respect to S_t (initially dS_T, the final-state gradient):
//     dS  += q do^T;             dq = S_t do
//     du   = dS^T k;             dk = dS u + S' dw,   dw = -beta du
//     dbeta = du . (v - w);      dv = beta du
//     dS' = dS + k dw^T;         dg = rowsum(dS' o S')
//     dS_{t-1} = Diag(a) dS'     (dS_0 is the initial-state gradient)
// Both directions are separable by state column: column c of S and of dS
// needs only k, q, a, beta and v_c, do_c.  So each warp owns 4 columns and
// runs on its own, except that the row sums over columns (dq, dk, dg,
// dbeta) meet per token in shared memory across the CTA's eight warps and
// leave as per-CTA partials, which a second kernel adds up in a fixed order.
//
// Per warp: a forward pass over the sequence storing its columns of the
// state at the start of every 8-token block, then blocks in reverse: the
// block's entering states are recomputed from the checkpoint into shared
// memory and the backward runs over them.  Lane l holds rows l * RPL ..
// l * RPL + RPL - 1 (RPL = DK / 32) of the warp's 4 columns.  Token rows are
// staged once per CTA.  All arithmetic is fp32.
#include "common.cuh"
#include "kernels.h"

namespace kda {
namespace {

constexpr int BT = 8;        // tokens per recomputed block
constexpr int TW = 4;        // state columns per warp
constexpr int NW = 8;        // warps per CTA
constexpr int CW = TW * NW;  // state columns per CTA

template <int DK, typename Tin>
struct BwdCfg {
    static constexpr int RPL = DK / 32;                      // rows per lane
    static constexpr int RK = DK * (int)sizeof(Tin);         // k or q row bytes
    static constexpr int RV = CW * (int)sizeof(Tin);         // v or do bytes of the CTA's columns
    // staged token: k, q (Tin), g (fp32), v, do (Tin, the CTA's columns), beta
    static constexpr int OK_ = 0, OQ = RK, OG = 2 * RK, OV = 2 * RK + DK * 4, OD = OV + RV,
                         OB = OD + RV;
    static constexpr int TOK = ((OB + 16 + 15) / 16) * 16;
    static constexpr int STAGE = BT * TOK;
    static constexpr int BUFW = BT * DK * TW * 4;            // a warp's entering states of a block
    static constexpr int OFF_STAGE = NW * BUFW;
    static constexpr int OFF_RED = OFF_STAGE + 2 * STAGE;    // [2][3][NW][DK] row partials
    static constexpr int OFF_REDB = OFF_RED + 2 * 3 * NW * DK * 4;   // [2][NW] dbeta partials
    static constexpr int SMEM = OFF_REDB + 2 * NW * 4;
    static_assert(RPL * 32 == DK && RV % 16 == 0 && RK % 16 == 0 && OFF_RED % 16 == 0, "tiling");
};

__device__ __forceinline__ void cp16z(void *dst, const void *src, bool ok) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_u32(dst)), "l"(src),
                 "r"(ok ? 16 : 0));
}
__device__ __forceinline__ void cp4z(void *dst, const void *src, bool ok) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n" ::"r"(smem_u32(dst)), "l"(src),
                 "r"(ok ? 4 : 0));
}
template <int N>
__device__ __forceinline__ void load_f(const float *p, float (&x)[N]) {
    if constexpr (N % 4 == 0) {
#pragma unroll
        for (int i = 0; i < N; i += 4) {
            const float4 t = *reinterpret_cast<const float4 *>(p + i);
            x[i] = t.x; x[i + 1] = t.y; x[i + 2] = t.z; x[i + 3] = t.w;
        }
    } else {
#pragma unroll
        for (int i = 0; i < N; i += 2) {
            const float2 t = *reinterpret_cast<const float2 *>(p + i);
            x[i] = t.x; x[i + 1] = t.y;
        }
    }
}
template <int N>
__device__ __forceinline__ void load_f(const __nv_bfloat16 *p, float (&x)[N]) {
    if constexpr (N % 4 == 0) {
#pragma unroll
        for (int i = 0; i < N; i += 4) {
            const uint2 t = *reinterpret_cast<const uint2 *>(p + i);
            const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162 *>(&t.x);
            const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162 *>(&t.y);
            x[i] = __low2float(lo); x[i + 1] = __high2float(lo);
            x[i + 2] = __low2float(hi); x[i + 3] = __high2float(hi);
        }
    } else {
#pragma unroll
        for (int i = 0; i < N; i += 2) {
            const __nv_bfloat162 t = *reinterpret_cast<const __nv_bfloat162 *>(p + i);
            x[i] = __low2float(t); x[i + 1] = __high2float(t);
        }
    }
}

}  // namespace

template <int DK, typename Tin>
__global__ void __launch_bounds__(NW * 32, 1)
recurrent_bwd_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
                     const float *__restrict__ g, const float *__restrict__ beta,
                     const float *__restrict__ s0, const Tin *__restrict__ dout,
                     const float *__restrict__ dsT, float *__restrict__ dv_out,
                     float *__restrict__ ds0, float *__restrict__ ckpt, float *__restrict__ part,
                     int T, int H, int DV)
{
    using C = BwdCfg<DK, Tin>;
    constexpr int RPL = C::RPL;
    extern __shared__ __align__(128) unsigned char sm[];
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const int ct = blockIdx.x, h = blockIdx.y, n = blockIdx.z;
    const int nct = gridDim.x;                          // CTA column tiles
    const int col0 = ct * CW + w * TW;                  // this warp's first state column
    const int r0 = lane * RPL;                          // this lane's first row
    const int nblk = (T + BT - 1) / BT;
    const size_t NTH = (size_t)gridDim.z * T * H;       // tokens x heads, all sequences
    float *ck = ckpt + (((size_t)n * H + h) * (nct * NW) + ct * NW + w) * (size_t)nblk * DK * TW;
    float *buf = reinterpret_cast<float *>(sm + w * C::BUFW);
    float *red = reinterpret_cast<float *>(sm + C::OFF_RED);
    float *redb = reinterpret_cast<float *>(sm + C::OFF_REDB);
    auto row_of = [&](int t) -> size_t { return ((size_t)n * T + t) * H + h; };

    // stage the tokens of block b into stage buffer sb (all threads, one cp.async group)
    auto stage = [&](int b, int sb) {
        unsigned char *st0 = sm + C::OFF_STAGE + sb * C::STAGE;
        const int t0 = b * BT, nt = min(BT, T - t0);
        constexpr int PK = C::RK / 16, PG = DK * 4 / 16, PV = C::RV / 16;
        constexpr int PER = 2 * PK + PG + 2 * PV + 1;
        for (int c = tid; c < BT * PER; c += NW * 32) {
            const int i = c / PER, r = c - i * PER;
            const bool ok = i < nt;
            const size_t row = row_of(ok ? t0 + i : t0);
            unsigned char *st = st0 + i * C::TOK;
            if (r < PK)
                cp16z(st + C::OK_ + 16 * r, reinterpret_cast<const unsigned char *>(k + row * DK) + 16 * r, ok);
            else if (r < 2 * PK)
                cp16z(st + C::OQ + 16 * (r - PK), reinterpret_cast<const unsigned char *>(q + row * DK) + 16 * (r - PK), ok);
            else if (r < 2 * PK + PG)
                cp16z(st + C::OG + 16 * (r - 2 * PK), reinterpret_cast<const unsigned char *>(g + row * DK) + 16 * (r - 2 * PK), ok);
            else if (r < 2 * PK + PG + PV)
                cp16z(st + C::OV + 16 * (r - 2 * PK - PG),
                      reinterpret_cast<const unsigned char *>(v + row * DV + ct * CW) + 16 * (r - 2 * PK - PG), ok);
            else if (r < 2 * PK + PG + 2 * PV)
                cp16z(st + C::OD + 16 * (r - 2 * PK - PG - PV),
                      reinterpret_cast<const unsigned char *>(dout + row * DV + ct * CW) + 16 * (r - 2 * PK - PG - PV), ok);
            else
                cp4z(st + C::OB, beta + row, ok);
        }
        cp_async_commit();
    };
    struct Tok { float k[RPL], q[RPL], a[RPL], v[TW], d[TW], b; };
    auto token = [&](int sb, int i, Tok &x) {
        const unsigned char *st = sm + C::OFF_STAGE + sb * C::STAGE + i * C::TOK;
        load_f<RPL>(reinterpret_cast<const Tin *>(st + C::OK_) + r0, x.k);
        load_f<RPL>(reinterpret_cast<const Tin *>(st + C::OQ) + r0, x.q);
        float gg[RPL];
        load_f<RPL>(reinterpret_cast<const float *>(st + C::OG) + r0, gg);
#pragma unroll
        for (int r = 0; r < RPL; ++r) x.a[r] = expf(gg[r]);
        load_f<TW>(reinterpret_cast<const Tin *>(st + C::OV) + w * TW, x.v);
        load_f<TW>(reinterpret_cast<const Tin *>(st + C::OD) + w * TW, x.d);
        x.b = *reinterpret_cast<const float *>(st + C::OB);
    };
    auto colsum = [&](float (&p)[TW]) {                  // over all rows: the whole warp
#pragma unroll
        for (int o = 1; o < 32; o <<= 1)
#pragma unroll
            for (int j = 0; j < TW; ++j) p[j] += __shfl_xor_sync(0xffffffffu, p[j], o);
    };
    // one forward step; w = S'^T k of the warp's columns is returned
    auto fwd = [&](float (&s)[RPL][TW], const Tok &x, float (&wv)[TW]) {
#pragma unroll
        for (int j = 0; j < TW; ++j) wv[j] = 0.f;
#pragma unroll
        for (int r = 0; r < RPL; ++r)
#pragma unroll
            for (int j = 0; j < TW; ++j) {
                s[r][j] *= x.a[r];
                wv[j] = fmaf(x.k[r], s[r][j], wv[j]);
            }
        colsum(wv);
#pragma unroll
        for (int j = 0; j < TW; ++j) {
            const float u = x.b * (x.v[j] - wv[j]);
#pragma unroll
            for (int r = 0; r < RPL; ++r) s[r][j] = fmaf(x.k[r], u, s[r][j]);
        }
    };
    auto ld_state = [&](const float *p, float (&s)[RPL][TW]) {   // [DK][TW] fp32
#pragma unroll
        for (int r = 0; r < RPL; ++r) load_f<TW>(p + (size_t)(r0 + r) * TW, s[r]);
    };
    auto st_state = [&](float *p, const float (&s)[RPL][TW]) {
#pragma unroll
        for (int r = 0; r < RPL; ++r)
            *reinterpret_cast<float4 *>(p + (size_t)(r0 + r) * TW) = make_float4(s[r][0], s[r][1], s[r][2], s[r][3]);
    };

    // ---- forward pass with a checkpoint at the start of every block ----
    float s[RPL][TW];
#pragma unroll
    for (int r = 0; r < RPL; ++r) {
        if (s0) load_f<TW>(s0 + (((size_t)n * H + h) * DK + r0 + r) * DV + col0, s[r]);
        else for (int j = 0; j < TW; ++j) s[r][j] = 0.f;
    }
    if (nblk > 0) stage(0, 0);
    for (int b = 0; b < nblk; ++b) {
        cp_async_wait<0>();
        __syncthreads();                                 // block b staged; block b - 1 done by all
        if (b + 1 < nblk) stage(b + 1, (b + 1) & 1);
        st_state(ck + (size_t)b * DK * TW, s);
        const int nt = min(BT, T - b * BT);
        for (int i = 0; i < nt; ++i) {
            Tok x;
            token(b & 1, i, x);
            float wv[TW];
            fwd(s, x, wv);
        }
    }
    cp_async_wait<0>();
    __syncthreads();

    // ---- backward over the blocks in reverse ----
    float ds[RPL][TW];
#pragma unroll
    for (int r = 0; r < RPL; ++r) {
        if (dsT) load_f<TW>(dsT + (((size_t)n * H + h) * DK + r0 + r) * DV + col0, ds[r]);
        else for (int j = 0; j < TW; ++j) ds[r][j] = 0.f;
    }
    float *pdq = part + (size_t)ct * NTH * DK;           // [3][CTA tile][token, head][DK]
    float *pdk = part + (size_t)(nct + ct) * NTH * DK;
    float *pdg = part + (size_t)(2 * nct + ct) * NTH * DK;
    float *pdb = part + (size_t)3 * nct * NTH * DK + (size_t)ct * NTH;
    int par = 0;                                         // parity of the reduction buffers
    if (nblk > 0) stage(nblk - 1, (nblk - 1) & 1);
    for (int b = nblk - 1; b >= 0; --b) {
        const int sb = b & 1, nt = min(BT, T - b * BT);
        cp_async_wait<0>();
        __syncthreads();                                 // block b staged; block b + 1 done by all
        if (b > 0) stage(b - 1, (b - 1) & 1);
        // entering state of every token of the block, from the checkpoint, and
        // each token's w = S'^T k (every lane holds its warp's four columns)
        ld_state(ck + (size_t)b * DK * TW, s);
        float wk[BT][TW];
#pragma unroll
        for (int i = 0; i < BT; ++i) {
            if (i < nt) {
                st_state(buf + (size_t)i * DK * TW, s);
                Tok x;
                token(sb, i, x);
                fwd(s, x, wk[i]);
            }
        }
        __syncwarp();
#pragma unroll
        for (int i = BT - 1; i >= 0; --i) {
            if (i >= nt) continue;
            Tok x;
            token(sb, i, x);
            float sp[RPL][TW];
            ld_state(buf + (size_t)i * DK * TW, sp);
#pragma unroll
            for (int r = 0; r < RPL; ++r)
#pragma unroll
                for (int j = 0; j < TW; ++j) sp[r][j] *= x.a[r];           // S'
            const float (&wv)[TW] = wk[i];
            float u[TW], du[TW] = {};
#pragma unroll
            for (int j = 0; j < TW; ++j) u[j] = x.b * (x.v[j] - wv[j]);
            float dq[RPL], dk[RPL], dg[RPL];
#pragma unroll
            for (int r = 0; r < RPL; ++r) {
                float aq = 0.f, ak = 0.f;
#pragma unroll
                for (int j = 0; j < TW; ++j) {
                    const float st_ = fmaf(x.k[r], u[j], sp[r][j]);   // S_t
                    aq = fmaf(st_, x.d[j], aq);
                    ds[r][j] = fmaf(x.q[r], x.d[j], ds[r][j]);     // + q do^T
                    du[j] = fmaf(ds[r][j], x.k[r], du[j]);
                    ak = fmaf(ds[r][j], u[j], ak);
                }
                dq[r] = aq;
                dk[r] = ak;
            }
            colsum(du);
            float dbp = 0.f, dw[TW];
#pragma unroll
            for (int j = 0; j < TW; ++j) {
                dbp = fmaf(du[j], x.v[j] - wv[j], dbp);
                dw[j] = -x.b * du[j];
            }
#pragma unroll
            for (int r = 0; r < RPL; ++r) {
                float ak = dk[r], ag = 0.f;
#pragma unroll
                for (int j = 0; j < TW; ++j) {
                    ds[r][j] = fmaf(x.k[r], dw[j], ds[r][j]);      // dS'
                    ak = fmaf(sp[r][j], dw[j], ak);
                    ag = fmaf(ds[r][j], sp[r][j], ag);
                    ds[r][j] *= x.a[r];                            // dS_{t-1}
                }
                dk[r] = ak;
                dg[r] = ag;
            }
            // the CTA's row sums: the eight warps meet in shared memory
            float *rd = red + (size_t)par * 3 * NW * DK;
#pragma unroll
            for (int r = 0; r < RPL; ++r) {
                rd[(0 * NW + w) * DK + r0 + r] = dq[r];
                rd[(1 * NW + w) * DK + r0 + r] = dk[r];
                rd[(2 * NW + w) * DK + r0 + r] = dg[r];
            }
            if (lane == 0) redb[par * NW + w] = dbp;
            const size_t row = row_of(b * BT + i);
            if (lane == 0)
                *reinterpret_cast<float4 *>(dv_out + row * DV + col0) =
                    make_float4(x.b * du[0], x.b * du[1], x.b * du[2], x.b * du[3]);
            __syncthreads();
            for (int x = tid; x <= 3 * DK; x += NW * 32) {
                float acc = 0.f;
                if (x < 3 * DK) {
                    const int qi = x / DK, rr = x - qi * DK;
#pragma unroll
                    for (int ww = 0; ww < NW; ++ww) acc += rd[(qi * NW + ww) * DK + rr];
                    (qi == 0 ? pdq : qi == 1 ? pdk : pdg)[row * DK + rr] = acc;
                } else {
#pragma unroll
                    for (int ww = 0; ww < NW; ++ww) acc += redb[par * NW + ww];
                    pdb[row] = acc;
                }
            }
            par ^= 1;
        }
    }
    if (ds0) {
#pragma unroll
        for (int r = 0; r < RPL; ++r)
            *reinterpret_cast<float4 *>(ds0 + (((size_t)n * H + h) * DK + r0 + r) * DV + col0) =
                make_float4(ds[r][0], ds[r][1], ds[r][2], ds[r][3]);
    }
}

// dq, dk, dg, dbeta = the sum of the CTA tiles' partials, tile 0 first
__global__ void bwd_reduce_kernel(const float *__restrict__ part, float *__restrict__ dq,
                                  float *__restrict__ dk, float *__restrict__ dg,
                                  float *__restrict__ db, size_t nrow, int DK, int ntiles)
{
    const size_t nel = nrow * DK;
    for (size_t x = blockIdx.x * (size_t)blockDim.x + threadIdx.x; x < 3 * nel + nrow;
         x += (size_t)gridDim.x * blockDim.x) {
        float acc = 0.f;
        if (x < 3 * nel) {
            const size_t which = x / nel, e = x - which * nel;
            for (int t = 0; t < ntiles; ++t) acc += part[((size_t)which * ntiles + t) * nel + e];
            (which == 0 ? dq : which == 1 ? dk : dg)[e] = acc;
        } else {
            const size_t e = x - 3 * nel;
            for (int t = 0; t < ntiles; ++t) acc += part[(size_t)3 * ntiles * nel + (size_t)t * nrow + e];
            db[e] = acc;
        }
    }
}

size_t recurrent_bwd_workspace(int B, int T, int H, int dk, int dv) {
    const size_t nct = (size_t)dv / CW, nblk = ((size_t)T + BT - 1) / BT;
    const size_t nrow = (size_t)B * T * H;
    const size_t ck = (size_t)B * H * (nct * NW) * nblk * dk * TW * 4;
    const size_t pt = (3 * nct * nrow * dk + nct * nrow) * 4;
    return ((ck + 255) & ~(size_t)255) + pt;
}

template <int DK, typename Tin>
static cudaError_t launch_bwd_t(const void *q, const void *k, const void *v, const float *g,
                                const float *beta, const float *s0, const void *dout,
                                const float *dsT, float *dq, float *dk, float *dv, float *dg,
                                float *db, float *ds0, void *ws, int B, int T, int H, int DV,
                                cudaStream_t st)
{
    using C = BwdCfg<DK, Tin>;
    auto kern = recurrent_bwd_kernel<DK, Tin>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    const size_t nct = (size_t)DV / CW, nblk = ((size_t)T + BT - 1) / BT;
    const size_t ck = (size_t)B * H * (nct * NW) * nblk * DK * TW * 4;
    float *ckpt = (float *)ws;
    float *part = (float *)((unsigned char *)ws + ((ck + 255) & ~(size_t)255));
    dim3 grid((unsigned)nct, H, B);
    kern<<<grid, NW * 32, C::SMEM, st>>>((const Tin *)q, (const Tin *)k, (const Tin *)v, g, beta, s0,
                                         (const Tin *)dout, dsT, dv, ds0, ckpt, part, T, H, DV);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const size_t nrow = (size_t)B * T * H;
    const size_t total = 3 * nrow * DK + nrow;
    const int blocks = (int)((total + 255) / 256 < 148 * 16 ? (total + 255) / 256 : 148 * 16);
    if (blocks > 0)
        bwd_reduce_kernel<<<blocks, 256, 0, st>>>(part, dq, dk, dg, db, nrow, DK, (int)nct);
    return cudaGetLastError();
}

cudaError_t launch_recurrent_bwd(const void *q, const void *k, const void *v, const float *g,
                                 const float *beta, const float *s0, const void *dout,
                                 const float *dsT, float *dq, float *dk, float *dv, float *dg,
                                 float *db, float *ds0, void *ws, int B, int T, int H, int dk_,
                                 int dv_, bool bf16, cudaStream_t st)
{
    if (dk_ == 128)
        return bf16 ? launch_bwd_t<128, __nv_bfloat16>(q, k, v, g, beta, s0, dout, dsT, dq, dk, dv, dg, db, ds0, ws, B, T, H, dv_, st)
                    : launch_bwd_t<128, float>(q, k, v, g, beta, s0, dout, dsT, dq, dk, dv, dg, db, ds0, ws, B, T, H, dv_, st);
    if (dk_ == 64)
        return bf16 ? launch_bwd_t<64, __nv_bfloat16>(q, k, v, g, beta, s0, dout, dsT, dq, dk, dv, dg, db, ds0, ws, B, T, H, dv_, st)
                    : launch_bwd_t<64, float>(q, k, v, g, beta, s0, dout, dsT, dq, dk, dv, dg, db, ds0, ws, B, T, H, dv_, st);
    return cudaErrorInvalidValue;
}

}  // namespace kda

// recurrent_bwd.cu -- gradients of the KDA recurrence (training backward),
// one warp per (sequence, head, 16-column tile of the state).
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
// needs only k, q, a, beta and v_c, do_c.  So each warp owns 16 columns and
// never talks to another; the row sums over all columns (dq, dk, dg, dbeta)
// leave as per-tile partials that a second kernel adds up in a fixed order.
//
// Per warp: a forward pass over the sequence storing the state at the start
// of every 8-token block, then blocks in reverse: the block's entering
// states are recomputed from its checkpoint into shared memory and the
// backward runs over them.  Lane layout: lane = 2 rg + cg holds rows
// rg * RPL .. + RPL - 1 (RPL = DK / 16) and tile columns 8 cg .. 8 cg + 7.
// All arithmetic is fp32.
#include "common.cuh"
#include "kernels.h"

namespace kda {
namespace {

constexpr int BT = 8;        // tokens per recomputed block
constexpr int TW = 16;       // state columns per warp

template <int DK, typename Tin>
struct BwdCfg {
    static constexpr int RPL = DK / 16;                      // rows per lane
    static constexpr int RK = DK * (int)sizeof(Tin);         // k or q row bytes
    static constexpr int RV = TW * (int)sizeof(Tin);         // v or do tile bytes
    // staged token: k, q (Tin), g (fp32), v tile, do tile (Tin), beta
    static constexpr int OK_ = 0, OQ = RK, OG = 2 * RK, OV = 2 * RK + DK * 4, OD = OV + RV + 16,
                         OB = OD + RV + 16;
    static constexpr int TOK = ((OB + 16 + 15) / 16) * 16;
    static constexpr int STAGE = BT * TOK;
    static constexpr int BUF = BT * DK * TW * 4;             // the block's entering states
    static constexpr int SMEM = BUF + 2 * STAGE;
    static_assert(RPL * 16 == DK && RV % 16 == 0 && RK % 16 == 0, "tiling");
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
#pragma unroll
    for (int i = 0; i < N; i += 4) {
        const float4 t = *reinterpret_cast<const float4 *>(p + i);
        x[i] = t.x; x[i + 1] = t.y; x[i + 2] = t.z; x[i + 3] = t.w;
    }
}
template <int N>
__device__ __forceinline__ void load_f(const __nv_bfloat16 *p, float (&x)[N]) {
    static_assert(N % 4 == 0, "four elements at a time");
#pragma unroll
    for (int i = 0; i < N; i += 4) {
        const uint2 t = *reinterpret_cast<const uint2 *>(p + i);
        const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162 *>(&t.x);
        const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162 *>(&t.y);
        x[i] = __low2float(lo);
        x[i + 1] = __high2float(lo);
        x[i + 2] = __low2float(hi);
        x[i + 3] = __high2float(hi);
    }
}

}  // namespace

template <int DK, typename Tin>
__global__ void __launch_bounds__(32)
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
    const int lane = threadIdx.x, rg = lane >> 1, cg = lane & 1;
    const int tile = blockIdx.x, h = blockIdx.y, n = blockIdx.z;
    const int ntiles = gridDim.x;
    const int col0 = tile * TW + 8 * cg;                // this lane's first state column
    const int r0 = rg * RPL;                            // this lane's first row
    const int nblk = (T + BT - 1) / BT;
    const size_t NTH = (size_t)gridDim.z * T * H;       // tokens x heads, all sequences
    float *ck = ckpt + (((size_t)n * H + h) * ntiles + tile) * (size_t)nblk * DK * TW;
    float *buf = reinterpret_cast<float *>(sm);
    auto row_of = [&](int t) -> size_t { return ((size_t)n * T + t) * H + h; };

    // stage the tokens of block b into stage buffer sb (cp.async, one group)
    auto stage = [&](int b, int sb) {
        unsigned char *st0 = sm + C::BUF + sb * C::STAGE;
        const int t0 = b * BT, nt = min(BT, T - t0);
        constexpr int PK = C::RK / 16, PG = DK * 4 / 16, PV = C::RV / 16;
        constexpr int PER = 2 * PK + PG + 2 * PV + 1;
        for (int c = lane; c < BT * PER; c += 32) {
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
                      reinterpret_cast<const unsigned char *>(v + row * DV + tile * TW) + 16 * (r - 2 * PK - PG), ok);
            else if (r < 2 * PK + PG + 2 * PV)
                cp16z(st + C::OD + 16 * (r - 2 * PK - PG - PV),
                      reinterpret_cast<const unsigned char *>(dout + row * DV + tile * TW) + 16 * (r - 2 * PK - PG - PV), ok);
            else
                cp4z(st + C::OB, beta + row, ok);
        }
        cp_async_commit();
    };
    // the token's per-lane values
    struct Tok { float k[RPL], q[RPL], a[RPL], v[8], d[8], b; };
    auto token = [&](int sb, int i, Tok &x) {
        const unsigned char *st = sm + C::BUF + sb * C::STAGE + i * C::TOK;
        load_f<RPL>(reinterpret_cast<const Tin *>(st + C::OK_) + r0, x.k);
        load_f<RPL>(reinterpret_cast<const Tin *>(st + C::OQ) + r0, x.q);
        float gg[RPL];
        load_f<RPL>(reinterpret_cast<const float *>(st + C::OG) + r0, gg);
#pragma unroll
        for (int r = 0; r < RPL; ++r) x.a[r] = expf(gg[r]);
        load_f<8>(reinterpret_cast<const Tin *>(st + C::OV) + 8 * cg, x.v);
        load_f<8>(reinterpret_cast<const Tin *>(st + C::OD) + 8 * cg, x.d);
        x.b = *reinterpret_cast<const float *>(st + C::OB);
    };
    // column sums over all rows (lanes with the same cg)
    auto colsum = [&](float (&p)[8]) {
#pragma unroll
        for (int o = 2; o < 32; o <<= 1)
#pragma unroll
            for (int j = 0; j < 8; ++j) p[j] += __shfl_xor_sync(0xffffffffu, p[j], o);
    };
    // one forward step on the lane's block of the state
    auto fwd = [&](float (&s)[RPL][8], const Tok &x) {
        float w[8] = {};
#pragma unroll
        for (int r = 0; r < RPL; ++r)
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                s[r][j] *= x.a[r];
                w[j] = fmaf(x.k[r], s[r][j], w[j]);
            }
        colsum(w);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float u = x.b * (x.v[j] - w[j]);
#pragma unroll
            for (int r = 0; r < RPL; ++r) s[r][j] = fmaf(x.k[r], u, s[r][j]);
        }
    };
    auto ld_state = [&](const float *p, float (&s)[RPL][8]) {   // [DK][TW] fp32
#pragma unroll
        for (int r = 0; r < RPL; ++r) load_f<8>(p + (size_t)(r0 + r) * TW + 8 * cg, s[r]);
    };
    auto st_state = [&](float *p, const float (&s)[RPL][8]) {
#pragma unroll
        for (int r = 0; r < RPL; ++r) {
            float4 *d = reinterpret_cast<float4 *>(p + (size_t)(r0 + r) * TW + 8 * cg);
            d[0] = make_float4(s[r][0], s[r][1], s[r][2], s[r][3]);
            d[1] = make_float4(s[r][4], s[r][5], s[r][6], s[r][7]);
        }
    };

    // ---- forward pass with a checkpoint at the start of every block ----
    float s[RPL][8];
#pragma unroll
    for (int r = 0; r < RPL; ++r)
#pragma unroll
        for (int j = 0; j < 8; ++j)
            s[r][j] = s0 ? s0[(((size_t)n * H + h) * DK + r0 + r) * DV + col0 + j] : 0.f;
    if (nblk > 0) stage(0, 0);
    for (int b = 0; b < nblk; ++b) {
        cp_async_wait<0>();
        __syncwarp();
        if (b + 1 < nblk) stage(b + 1, (b + 1) & 1);
        st_state(ck + (size_t)b * DK * TW, s);
        const int nt = min(BT, T - b * BT);
        for (int i = 0; i < nt; ++i) {
            Tok x;
            token(b & 1, i, x);
            fwd(s, x);
        }
        __syncwarp();
    }
    cp_async_wait<0>();
    __syncwarp();

    // ---- backward over the blocks in reverse ----
    float ds[RPL][8];
#pragma unroll
    for (int r = 0; r < RPL; ++r)
#pragma unroll
        for (int j = 0; j < 8; ++j)
            ds[r][j] = dsT ? dsT[(((size_t)n * H + h) * DK + r0 + r) * DV + col0 + j] : 0.f;
    float *pdq = part + (size_t)tile * NTH * DK;          // [tile][token, head][DK]
    float *pdk = part + (size_t)(ntiles + tile) * NTH * DK;
    float *pdg = part + (size_t)(2 * ntiles + tile) * NTH * DK;
    float *pdb = part + (size_t)3 * ntiles * NTH * DK + (size_t)tile * NTH;
    if (nblk > 0) stage(nblk - 1, (nblk - 1) & 1);
    for (int b = nblk - 1; b >= 0; --b) {
        const int sb = b & 1, nt = min(BT, T - b * BT);
        cp_async_wait<0>();
        __syncwarp();
        if (b > 0) stage(b - 1, (b - 1) & 1);
        // entering state of every token of the block, from the checkpoint
        ld_state(ck + (size_t)b * DK * TW, s);
        for (int i = 0; i < nt; ++i) {
            st_state(buf + (size_t)i * DK * TW, s);
            if (i + 1 < nt) {
                Tok x;
                token(sb, i, x);
                fwd(s, x);
            }
        }
        __syncwarp();
        for (int i = nt - 1; i >= 0; --i) {
            Tok x;
            token(sb, i, x);
            float sp[RPL][8];
            ld_state(buf + (size_t)i * DK * TW, sp);
            float w[8] = {};
#pragma unroll
            for (int r = 0; r < RPL; ++r)
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    sp[r][j] *= x.a[r];                          // S'
                    w[j] = fmaf(x.k[r], sp[r][j], w[j]);
                }
            colsum(w);
            float u[8], du[8] = {};
#pragma unroll
            for (int j = 0; j < 8; ++j) u[j] = x.b * (x.v[j] - w[j]);
            float dq[RPL], dk1[RPL];
#pragma unroll
            for (int r = 0; r < RPL; ++r) {
                float aq = 0.f, ak = 0.f;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float st_ = fmaf(x.k[r], u[j], sp[r][j]);   // S_t
                    aq = fmaf(st_, x.d[j], aq);
                    ds[r][j] = fmaf(x.q[r], x.d[j], ds[r][j]);     // + q do^T
                    du[j] = fmaf(ds[r][j], x.k[r], du[j]);
                    ak = fmaf(ds[r][j], u[j], ak);
                }
                dq[r] = aq;
                dk1[r] = ak;
            }
            colsum(du);
            float dbp = 0.f, dw[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                dbp = fmaf(du[j], x.v[j] - w[j], dbp);
                dw[j] = -x.b * du[j];
            }
            float dk[RPL], dg[RPL];
#pragma unroll
            for (int r = 0; r < RPL; ++r) {
                float ak = dk1[r], ag = 0.f;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    ds[r][j] = fmaf(x.k[r], dw[j], ds[r][j]);      // dS'
                    ak = fmaf(sp[r][j], dw[j], ak);
                    ag = fmaf(ds[r][j], sp[r][j], ag);
                    ds[r][j] *= x.a[r];                            // dS_{t-1}
                }
                dk[r] = ak;
                dg[r] = ag;
            }
            // the tile's row sums: the two column halves meet
#pragma unroll
            for (int r = 0; r < RPL; ++r) {
                dq[r] += __shfl_xor_sync(0xffffffffu, dq[r], 1);
                dk[r] += __shfl_xor_sync(0xffffffffu, dk[r], 1);
                dg[r] += __shfl_xor_sync(0xffffffffu, dg[r], 1);
            }
            dbp += __shfl_xor_sync(0xffffffffu, dbp, 1);
            const size_t row = row_of(b * BT + i);
            if (cg == 0) {
#pragma unroll
                for (int r = 0; r < RPL; r += 4) {
                    *reinterpret_cast<float4 *>(pdq + row * DK + r0 + r) = make_float4(dq[r], dq[r + 1], dq[r + 2], dq[r + 3]);
                    *reinterpret_cast<float4 *>(pdk + row * DK + r0 + r) = make_float4(dk[r], dk[r + 1], dk[r + 2], dk[r + 3]);
                    *reinterpret_cast<float4 *>(pdg + row * DK + r0 + r) = make_float4(dg[r], dg[r + 1], dg[r + 2], dg[r + 3]);
                }
            }
            if (rg == 0) {
                float4 *d = reinterpret_cast<float4 *>(dv_out + row * DV + col0);
                d[0] = make_float4(x.b * du[0], x.b * du[1], x.b * du[2], x.b * du[3]);
                d[1] = make_float4(x.b * du[4], x.b * du[5], x.b * du[6], x.b * du[7]);
            }
            if (lane == 0) pdb[row] = dbp;
        }
        __syncwarp();
    }
    if (ds0) {
#pragma unroll
        for (int r = 0; r < RPL; ++r) {
            float4 *d = reinterpret_cast<float4 *>(ds0 + (((size_t)n * H + h) * DK + r0 + r) * DV + col0);
            d[0] = make_float4(ds[r][0], ds[r][1], ds[r][2], ds[r][3]);
            d[1] = make_float4(ds[r][4], ds[r][5], ds[r][6], ds[r][7]);
        }
    }
}

// dq, dk, dg, dbeta = the sum of the tiles' partials, tile 0 first
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
    const size_t ntiles = (size_t)dv / TW, nblk = ((size_t)T + BT - 1) / BT;
    const size_t nrow = (size_t)B * T * H;
    const size_t ck = (size_t)B * H * ntiles * nblk * dk * TW * 4;
    const size_t pt = (3 * ntiles * nrow * dk + ntiles * nrow) * 4;
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
    const size_t ntiles = (size_t)DV / TW, nblk = ((size_t)T + BT - 1) / BT;
    const size_t ck = (size_t)B * H * ntiles * nblk * DK * TW * 4;
    float *ckpt = (float *)ws;
    float *part = (float *)((unsigned char *)ws + ((ck + 255) & ~(size_t)255));
    dim3 grid((unsigned)ntiles, H, B);
    kern<<<grid, 32, C::SMEM, st>>>((const Tin *)q, (const Tin *)k, (const Tin *)v, g, beta, s0,
                                    (const Tin *)dout, dsT, dv, ds0, ckpt, part, T, H, DV);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const size_t nrow = (size_t)B * T * H;
    const size_t total = 3 * nrow * DK + nrow;
    const int blocks = (int)((total + 255) / 256 < 148 * 16 ? (total + 255) / 256 : 148 * 16);
    if (blocks > 0)
        bwd_reduce_kernel<<<blocks, 256, 0, st>>>(part, dq, dk, dg, db, nrow, DK, (int)ntiles);
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

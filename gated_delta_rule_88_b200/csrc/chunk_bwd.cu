// chunk_bwd.cu -- per-(chunk, head) pass of the chunked KDA backward (bf16,
// dk = dv = 128, C = 64) on tcgen05.
//
// Given, per (chunk, head), the state S entering the chunk and V_new (forward
// chain images) and dS' (gradient of the state leaving the chunk) and dV_new
// (reverse chain images), and dO, this CTA recomputes the forms, A and
// T = (I + A)^-1 (chunk-start exponent reference, as in the prep) and forms
//   dQg = dO S^T + dP Kinv            dP   = tril0(dO V_new^T)
//   dW  = -dV_new S^T                 dKt  = V_new dS'^T
//   dT  = dV_new (bV)^T + dW (bKg)^T  dA   = tril_-1(-T^T dT T^T)
//   dbV = T^T dV_new                  dbKg = T^T dW + dA Kinv
//   dKinv = dA^T bKg + dP^T Qg        de^{G_C} = rowsum(S o dS')
// then dq, dk, dv, dbeta and dG per token and channel, and dg as the reverse
// cumsum of dG inside the chunk (the last row also collects the G_C terms).
// Products are M = 64 tcgen05 MMAs; two M = 64 accumulators share a column
// range, one on TMEM lanes 0-15 of each sub-partition (+0), one on lanes
// 16-31 (+16), so a warp's lane l reads row 16 (warp % 4) + (l % 16) of the
// +0 tile (l < 16) or of the +16 tile (l >= 16).
//
// TMEM columns (512, one CTA per SM):
//   0-127   D_Q (+0)     D_W (+16)
//   128-255 D_Kt (+0)    D_Kinv (+16)
//   256-319 D_P (+0)     D_T (+16)     (first: MMA-AP, M = 128)
//   320-383 X (+0)       Y (+16)
//   384-511 D_bV (+0)    D_bKg (+16)
#include "chunk_ws.h"
#include "common.cuh"
#include "kernels.h"
#include "prep_common.cuh"
#include "sm100.cuh"

namespace kda {
using namespace prep;
namespace {
using namespace sm100;

// 128-byte swizzle offset of (row r, channel c in 0..63) in a 64-channel block
__device__ __forceinline__ int sw(int r, int c) {
    return r * 128 + ((((c >> 3) ^ (r & 7))) << 4) + ((c & 7) << 1);
}
constexpr float RANGE2 = 80.f * 1.4426950408889634f;   // e^{+-80}, in log2 units
// 256-bit global store (32-byte aligned address)
__device__ __forceinline__ void st_v8(float *p, const float *v) {
    asm volatile("st.global.v8.f32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};\n" ::"l"(p), "f"(v[0]), "f"(v[1]), "f"(v[2]),
                 "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7])
                 : "memory");
}

namespace bl {
constexpr int KQ = 0;            // [k -> bKg : 64 rows][q -> Qg : 64 rows] per 64-ch block (16 KB); finale: dG fp32
constexpr int KI = 32768;        // Kinv, blocks of 8 KB
constexpr int V = 49152;         // v -> bV, blocks of 8 KB
constexpr int DO = 65536;        // dO (TMA), blocks of 8 KB
constexpr int VN = 81920;        // V_new image
constexpr int DVN = 98304;       // dV_new image
constexpr int TB = 114688;       // T bf16 (64 rows x 128 B)
constexpr int G = 122880;        // G in log2 units, fp32 [64][128] (g lands here by TMA)
constexpr int WA = 155648;       // 64 KB work area
constexpr int AM = WA, TM = WA + 16384, AD = WA + 32768, GS = WA + 49152;   // phase 1
constexpr int S = WA, DS = WA + 32768;                                        // phase 2a
constexpr int DW = WA, DP = WA + 16384, DT = WA + 24576, XI = WA + 32768, DA = WA + 40960;
constexpr int BETA = WA + 65536;                 // 64 floats
constexpr int DEGC = BETA + 256;                 // 128 floats: rowsum(S o dS')
constexpr int KTS = DEGC + 512;                  // [4][128] floats: sum_i dKt o Kt per row group
constexpr int DB = KTS + 2048;                   // [2][64] floats: dbeta per channel half
constexpr int BAR = DB + 512;                    // 6 mbarriers
constexpr int TSLOT = BAR + 48;
constexpr int BYTES = TSLOT + 16;
constexpr uint32_t TX_QKV = 6 * 8192, TX_G = 64 * 128 * 4, TX_IN2 = 2 * 8192 + 2 * 16384, TX_IN3 = 2 * 32768;
}  // namespace bl

__host__ __device__ constexpr uint32_t idesc_g(int M, int N, bool a_mn, bool b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
// K-major SW128 operand, 64-column blocks `bs` bytes apart: offset of K step kk (16 elements)
__device__ __forceinline__ uint32_t kmaj(int kk, uint32_t bs) { return ((kk >> 2) * bs + (kk & 3) * 32) >> 4; }
// MN-major SW128 operand: K step kk (two 8-row groups)
__device__ __forceinline__ uint32_t mnmaj(int kk) { return (kk * 2048) >> 4; }
// byte offset of (row r, column c) in a K-major SW128 image with 64-column blocks `bs` apart
__device__ __forceinline__ uint32_t img_off(int r, int c, uint32_t bs) {
    return (c >> 6) * bs + r * 128 + ((((c & 63) >> 3) ^ (r & 7)) << 4) + ((c & 7) << 1);
}
// fp32 [64][128] tile with the column XOR-swizzled by the row: 16 lanes on
// 16 consecutive rows and one column hit 16 different banks
__device__ __forceinline__ int gsw(int r, int c) { return r * 128 + (c ^ ((r & 15) << 1)); }
// 8 floats -> one 16-byte chunk of bf16
__device__ __forceinline__ uint4 pack8(const float *x, float s) {
    return make_uint4(pack_bf16(s * x[0], s * x[1]), pack_bf16(s * x[2], s * x[3]), pack_bf16(s * x[4], s * x[5]),
                      pack_bf16(s * x[6], s * x[7]));
}

__global__ void __launch_bounds__(NT, 1)
chunk_bwd_local_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                       const __grid_constant__ CUtensorMap tm_do,
                       const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                       const __nv_bfloat16 *__restrict__ v, const float *__restrict__ beta,
                       const int32_t *__restrict__ cu, const int32_t *__restrict__ coff, int N, int T,
                       int total_T, int H, int cps,
                       const unsigned char *__restrict__ s_img, const unsigned char *__restrict__ v_img,
                       const unsigned char *__restrict__ dsp_img, const unsigned char *__restrict__ dvn_img,
                       float *__restrict__ dq, float *__restrict__ dk, float *__restrict__ dv,
                       float *__restrict__ dg, float *__restrict__ dbeta, int v8, int *__restrict__ err)
{
    using namespace sm100;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int h = blockIdx.y, chunk = blockIdx.x;
    if (cu && chunk >= coff[N]) return;
    int len;
    long long t0;
    locate_chunk(chunk, cu, coff, N, T, total_T, cps, t0, len);
    const size_t slot = (size_t)chunk * H + h;

    uint64_t *bar_g = reinterpret_cast<uint64_t *>(sm + bl::BAR);
    uint64_t *bar_ld = bar_g + 1, *bar_in2 = bar_g + 2, *bar_in3 = bar_g + 3, *bar_mma = bar_g + 4;
    uint64_t *bar_fin = bar_g + 5;      // q, k, v again, for the finale
    uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + bl::TSLOT);
    float *bet = reinterpret_cast<float *>(sm + bl::BETA);
    float *degc = reinterpret_cast<float *>(sm + bl::DEGC);
    float *kts = reinterpret_cast<float *>(sm + bl::KTS);
    float *dbs = reinterpret_cast<float *>(sm + bl::DB);
    float *G2 = reinterpret_cast<float *>(sm + bl::G);

    if (tid == 0) {
        for (int b = 0; b < 6; ++b) mbar_init(bar_g + b, 1);
        fence_mbar_init();
        const int tt = (int)t0;
        mbar_arrive_expect_tx(bar_g, bl::TX_G);
        tma_load_3d(sm + bl::G, &tm_g, 0, h, tt, bar_g);
        mbar_arrive_expect_tx(bar_ld, bl::TX_QKV);
        mbar_arrive_expect_tx(bar_in2, bl::TX_IN2);
#pragma unroll
        for (int b = 0; b < 2; ++b) {
            tma_load_3d(sm + bl::KQ + b * 16384, &tm_k, 64 * b, h, tt, bar_ld);
            tma_load_3d(sm + bl::KQ + b * 16384 + 8192, &tm_q, 64 * b, h, tt, bar_ld);
            tma_load_3d(sm + bl::V + b * 8192, &tm_v, 64 * b, h, tt, bar_ld);
            tma_load_3d(sm + bl::DO + b * 8192, &tm_do, 64 * b, h, tt, bar_in2);
        }
        bulk_g2s(sm + bl::VN, v_img + slot * 16384, 16384, bar_in2);
        bulk_g2s(sm + bl::DVN, dvn_img + slot * 16384, 16384, bar_in2);
    }
    if (tid < C) bet[tid] = tid < len ? beta[(size_t)(t0 + tid) * H + h] : 0.f;
    if (warp == 0) { tmem_alloc(tslot, 512); tmem_relinquish(); }
    bool ok = true;
    if (tid == 0) ok = mbar_wait(bar_g, 0);
    tc_fence_before();
    ok = __syncthreads_and(ok);
    tc_fence_after();
    const uint32_t tmem = *tslot;
    uint32_t mma_phase = 0;
    // one thread issues, commits and waits; everyone meets at the barrier
    auto mma_done = [&](bool okk) -> bool {
        if (tid == 0 && okk) okk = mbar_wait(bar_mma, mma_phase & 1);
        ++mma_phase;
        okk = __syncthreads_and(okk);
        tc_fence_after();
        return okk;
    };

    // ---- cumsum of g in log2 units (thread: sub-chunk I, channels c0, c0 + 1), range check ----
    const int I = tid >> 6, c0 = 2 * (tid & 63);
    bool bad = false;
    {
        constexpr float L2E = 1.4426950408889634f;
        float *gs = reinterpret_cast<float *>(sm + bl::GS);
        float2 Gv[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int r = 16 * I + i;
            Gv[i] = r < len ? *reinterpret_cast<const float2 *>(G2 + r * D + c0) : make_float2(0.f, 0.f);
        }
        Gv[0].x *= L2E; Gv[0].y *= L2E;
#pragma unroll
        for (int i = 1; i < 16; ++i) { Gv[i].x = fmaf(Gv[i].x, L2E, Gv[i - 1].x); Gv[i].y = fmaf(Gv[i].y, L2E, Gv[i - 1].y); }
        *reinterpret_cast<float2 *>(gs + I * D + c0) = Gv[15];
        __syncthreads();
        float2 GC = make_float2(0.f, 0.f), PF = make_float2(0.f, 0.f);
#pragma unroll
        for (int J = 0; J < 4; ++J) {
            const float2 sj = *reinterpret_cast<const float2 *>(gs + J * D + c0);
            if (J < I) { PF.x += sj.x; PF.y += sj.y; }
            GC.x += sj.x; GC.y += sj.y;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            Gv[i].x += PF.x; Gv[i].y += PF.y;
            bad |= !(fabsf(Gv[i].x) <= RANGE2 && fabsf(Gv[i].y) <= RANGE2 &&
                     GC.x - Gv[i].x <= RANGE2 && GC.y - Gv[i].y <= RANGE2);
            *reinterpret_cast<float2 *>(G2 + gsw(16 * I + i, c0)) = Gv[i];
        }
    }
    if (tid == 0 && ok) ok = mbar_wait(bar_ld, 0);
    ok = __syncthreads_and(ok);
    bad = __syncthreads_or(bad);
    if (bad) {
        // out of the chunk-start exponent range: reported, gradients not written
        if (tid == 0) set_device_error(err, kErrBwdRange);
        ok = false;
    }

    // ---- forms: k -> beta k e^G, q -> q e^G (in place), k e^{-G} -> KI, v -> beta v ----
    if (ok) {
        const int cb = c0 >> 6, cc = c0 & 63;
        unsigned char *kq = sm + bl::KQ + cb * 16384;
        unsigned char *ki = sm + bl::KI + cb * 8192;
        unsigned char *vv = sm + bl::V + cb * 8192;
#pragma unroll 4
        for (int i = 0; i < 16; ++i) {
            const int r = 16 * I + i;
            const int o = sw(r, cc);
            const float2 Gi = *reinterpret_cast<const float2 *>(G2 + gsw(r, c0));
            const float2 eg = make_float2(ex2_approx(Gi.x), ex2_approx(Gi.y));
            const float2 em = make_float2(ex2_approx(-Gi.x), ex2_approx(-Gi.y));
            float2 qf = bf16x2_to_float2(*reinterpret_cast<const uint32_t *>(kq + 8192 + o));
            float2 kf = bf16x2_to_float2(*reinterpret_cast<const uint32_t *>(kq + o));
            float2 vf = bf16x2_to_float2(*reinterpret_cast<const uint32_t *>(vv + o));
            if (r >= len) { qf = kf = vf = make_float2(0.f, 0.f); }
            const float br = bet[r];
            *reinterpret_cast<uint32_t *>(kq + 8192 + o) = pack_bf16(qf.x * eg.x, qf.y * eg.y);
            *reinterpret_cast<uint32_t *>(kq + o) = pack_bf16(br * kf.x * eg.x, br * kf.y * eg.y);
            *reinterpret_cast<uint32_t *>(ki + o) = pack_bf16(kf.x * em.x, kf.y * em.y);
            *reinterpret_cast<uint32_t *>(vv + o) = pack_bf16(br * vf.x, br * vf.y);
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    const uint32_t sb = smem_u32(sm);
    const uint32_t L16 = 16u << 16;                     // +16 lane tile

    // ---- MMA-AP: [bKg ; Qg] Kinv^T -> cols 256-319 (A on lanes 0-63) ----
    if (tid == 0 && ok) {
        tc_fence_after();
        constexpr uint32_t ID = idesc_g(128, 64, false, false);
        const DescParts a = smem_desc_parts(sb + bl::KQ, 16, 1024, 2);
        const DescParts b = smem_desc_parts(sb + bl::KI, 16, 1024, 2);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
            umma_bf16_p(tmem + 256, a.lo + kmaj(kk, 16384), a.hi, b.lo + kmaj(kk, 8192), b.hi, ID, kk > 0);
        umma_commit(bar_mma);
    }
    ok = mma_done(ok);

    // ---- A (j < i) -> fp32 Am and the padded diagonal copy; T; T -> bf16 ----
    float *Am = reinterpret_cast<float *>(sm + bl::AM);
    float *Tm = reinterpret_cast<float *>(sm + bl::TM);
    float *Ad = reinterpret_cast<float *>(sm + bl::AD);
    if (ok && warp < 2) {
        float x[64];
        const uint32_t ta = tmem + 256 + ((uint32_t)(warp * 32) << 16);
        tmem_ld32(ta, *reinterpret_cast<float (*)[32]>(&x[0]));
        tmem_ld32(ta + 32, *reinterpret_cast<float (*)[32]>(&x[32]));
        tmem_wait_ld();
        const int i = warp * 32 + lane;
#pragma unroll
        for (int j4 = 0; j4 < 16; ++j4) {
            float4 a4;
            a4.x = (4 * j4 < i) ? x[4 * j4] : 0.f;
            a4.y = (4 * j4 + 1 < i) ? x[4 * j4 + 1] : 0.f;
            a4.z = (4 * j4 + 2 < i) ? x[4 * j4 + 2] : 0.f;
            a4.w = (4 * j4 + 3 < i) ? x[4 * j4 + 3] : 0.f;
            *reinterpret_cast<float4 *>(Am + i * 64 + 4 * (j4 ^ (i & 7))) = a4;
        }
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
    }
    tc_fence_before();
    __syncthreads();
    if (ok) {
        form_T_padded_diag(Am, Ad, Tm, Ad, tid);
        const int i = tid >> 2, jq = tid & 3;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int jg = 2 * jq + hh;
            const float4 lo = *reinterpret_cast<const float4 *>(Tm + i * 64 + 4 * ((2 * jg) ^ (i & 7)));
            const float4 hi = *reinterpret_cast<const float4 *>(Tm + i * 64 + 4 * ((2 * jg + 1) ^ (i & 7)));
            *reinterpret_cast<uint4 *>(sm + bl::TB + i * 128 + ((jg ^ (i & 7)) << 4)) =
                make_uint4(pack_bf16(lo.x, lo.y), pack_bf16(lo.z, lo.w), pack_bf16(hi.x, hi.y), pack_bf16(hi.z, hi.w));
        }
    }
    fence_proxy_async_smem();
    __syncthreads();

    // ---- S and dS' images into the work area (A, T fp32 are dead) ----
    bool in3_issued = false;
    if (tid == 0 && ok) {
        in3_issued = true;
        mbar_arrive_expect_tx(bar_in3, bl::TX_IN3);
        bulk_g2s(sm + bl::S, s_img + slot * 32768, 32768, bar_in3);
        bulk_g2s(sm + bl::DS, dsp_img + slot * 32768, 32768, bar_in3);
        ok = mbar_wait(bar_in2, 0) && mbar_wait(bar_in3, 0);
    }
    ok = __syncthreads_and(ok);

    // ---- phase 2a products ----
    if (tid == 0 && ok) {
        tc_fence_after();
        constexpr uint32_t ID128 = idesc_g(64, 128, false, false), ID64 = idesc_g(64, 64, false, false);
        const DescParts a_do = smem_desc_parts(sb + bl::DO, 16, 1024, 2);
        const DescParts a_dvn = smem_desc_parts(sb + bl::DVN, 16, 1024, 2);
        const DescParts a_vn = smem_desc_parts(sb + bl::VN, 16, 1024, 2);
        const DescParts b_s = smem_desc_parts(sb + bl::S, 16, 1024, 2);
        const DescParts b_ds = smem_desc_parts(sb + bl::DS, 16, 1024, 2);
        const DescParts b_vn = smem_desc_parts(sb + bl::VN, 16, 1024, 2);
        const DescParts b_bv = smem_desc_parts(sb + bl::V, 16, 1024, 2);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)      // D_Q = dO S^T
            umma_bf16_p(tmem + 0, a_do.lo + kmaj(kk, 8192), a_do.hi, b_s.lo + kmaj(kk, 16384), b_s.hi, ID128, kk > 0);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)      // D_W = dV_new S^T  (= -dW)
            umma_bf16_p(tmem + L16, a_dvn.lo + kmaj(kk, 8192), a_dvn.hi, b_s.lo + kmaj(kk, 16384), b_s.hi, ID128, kk > 0);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)      // D_Kt = V_new dS'^T
            umma_bf16_p(tmem + 128, a_vn.lo + kmaj(kk, 8192), a_vn.hi, b_ds.lo + kmaj(kk, 16384), b_ds.hi, ID128, kk > 0);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)      // D_P = dO V_new^T
            umma_bf16_p(tmem + 256, a_do.lo + kmaj(kk, 8192), a_do.hi, b_vn.lo + kmaj(kk, 8192), b_vn.hi, ID64, kk > 0);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)      // D_T = dV_new (bV)^T
            umma_bf16_p(tmem + 256 + L16, a_dvn.lo + kmaj(kk, 8192), a_dvn.hi, b_bv.lo + kmaj(kk, 8192), b_bv.hi, ID64, kk > 0);
        umma_commit(bar_mma);
    }
    // de^{G_C} = rowsum(S o dS') from the bf16 images (two threads per channel row)
    if (ok) {
        const int c = tid >> 1, b = tid & 1;
        float s = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint32_t off = b * 16384 + c * 128 + ((j ^ (c & 7)) << 4);
            const uint4 xs = *reinterpret_cast<const uint4 *>(sm + bl::S + off);
            const uint4 xd = *reinterpret_cast<const uint4 *>(sm + bl::DS + off);
            const uint32_t ws_[4] = {xs.x, xs.y, xs.z, xs.w}, wd[4] = {xd.x, xd.y, xd.z, xd.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 a = bf16x2_to_float2(ws_[e]), d = bf16x2_to_float2(wd[e]);
                s = fmaf(a.x, d.x, fmaf(a.y, d.y, s));
            }
        }
        s += __shfl_xor_sync(0xffffffffu, s, 1);
        if (b == 0) degc[c] = s;
    }
    ok = mma_done(ok);
    // dO, V_new and beta v are dead: q, k and v come again (raw, by TMA) into
    // their places for the finale, while the products below run
    bool fin_issued = false;
    if (tid == 0 && ok) {
        fin_issued = true;
        mbar_arrive_expect_tx(bar_fin, bl::TX_QKV);
#pragma unroll
        for (int b = 0; b < 2; ++b) {
            tma_load_3d(sm + bl::DO + b * 8192, &tm_q, 64 * b, h, (int)t0, bar_fin);
            tma_load_3d(sm + bl::VN + b * 8192, &tm_k, 64 * b, h, (int)t0, bar_fin);
            tma_load_3d(sm + bl::V + b * 8192, &tm_v, 64 * b, h, (int)t0, bar_fin);
        }
    }

    // ---- readback: dW = -D_W (lanes +16, cols 0-127) -> DW image; dP = tril0(D_P) -> DP image ----
    const int sub = warp & 3, l16 = lane & 15, hi = lane >> 4;
    const int row = 16 * sub + l16;                    // token row of this lane's tile
    const uint32_t lane_base = (uint32_t)(32 * sub) << 16;
    if (ok) {
        if (warp < 4) {
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
                float x[32];
                tmem_ld32(tmem + lane_base + 32 * c4, x);
                tmem_wait_ld();
                if (hi) {
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        *reinterpret_cast<uint4 *>(sm + bl::DW + img_off(row, 32 * c4 + 8 * e, 8192)) = pack8(x + 8 * e, -1.f);
                }
            }
        } else {
#pragma unroll
            for (int c2 = 0; c2 < 2; ++c2) {
                float x[32];
                tmem_ld32(tmem + lane_base + 256 + 32 * c2, x);
                tmem_wait_ld();
                if (!hi) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) x[j] = (32 * c2 + j <= row) ? x[j] : 0.f;
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        *reinterpret_cast<uint4 *>(sm + bl::DP + img_off(row, 32 * c2 + 8 * e, 8192)) = pack8(x + 8 * e, 1.f);
                }
            }
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---- phase 2b: D_T += dW (bKg)^T; D_Q += dP Kinv; D_Kinv = dP^T Qg ----
    if (tid == 0 && ok) {
        tc_fence_after();
        const DescParts a_dw = smem_desc_parts(sb + bl::DW, 16, 1024, 2);
        const DescParts b_bkg = smem_desc_parts(sb + bl::KQ, 16, 1024, 2);
        const DescParts a_dp = smem_desc_parts(sb + bl::DP, 16, 1024, 2);
        const DescParts a_dpt = smem_desc_parts(sb + bl::DP, 16384, 1024, 2);
        const DescParts b_kinv = smem_desc_parts(sb + bl::KI, 8192, 1024, 2);
        const DescParts b_qg = smem_desc_parts(sb + bl::KQ + 8192, 16384, 1024, 2);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
            umma_bf16_p(tmem + 256 + L16, a_dw.lo + kmaj(kk, 8192), a_dw.hi, b_bkg.lo + kmaj(kk, 16384), b_bkg.hi,
                        idesc_g(64, 64, false, false), 1);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            umma_bf16_p(tmem + 0, a_dp.lo + kmaj(kk, 8192), a_dp.hi, b_kinv.lo + mnmaj(kk), b_kinv.hi,
                        idesc_g(64, 128, false, true), 1);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            umma_bf16_p(tmem + 128 + L16, a_dpt.lo + mnmaj(kk), a_dpt.hi, b_qg.lo + mnmaj(kk), b_qg.hi,
                        idesc_g(64, 128, true, true), kk > 0);
        umma_commit(bar_mma);
    }
    ok = mma_done(ok);

    // ---- dT (lanes +16, cols 256-319) -> DT image ----
    if (ok && warp >= 4) {
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2) {
            float x[32];
            tmem_ld32(tmem + lane_base + 256 + 32 * c2, x);
            tmem_wait_ld();
            if (hi) {
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    *reinterpret_cast<uint4 *>(sm + bl::DT + img_off(row, 32 * c2 + 8 * e, 8192)) = pack8(x + 8 * e, 1.f);
            }
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    // ---- X = dT T^T (cols 320-383, +0) ----
    if (tid == 0 && ok) {
        tc_fence_after();
        const DescParts a_dt = smem_desc_parts(sb + bl::DT, 16, 1024, 2);
        const DescParts b_t = smem_desc_parts(sb + bl::TB, 16, 1024, 2);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            umma_bf16_p(tmem + 320, a_dt.lo + kmaj(kk, 8192), a_dt.hi, b_t.lo + kmaj(kk, 8192), b_t.hi,
                        idesc_g(64, 64, false, false), kk > 0);
        umma_commit(bar_mma);
    }
    ok = mma_done(ok);
    if (ok && warp < 4) {
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2) {
            float x[32];
            tmem_ld32(tmem + lane_base + 320 + 32 * c2, x);
            tmem_wait_ld();
            if (!hi) {
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    *reinterpret_cast<uint4 *>(sm + bl::XI + img_off(row, 32 * c2 + 8 * e, 8192)) = pack8(x + 8 * e, 1.f);
            }
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    // ---- Y = T^T X (cols 320-383, +16) ----
    if (tid == 0 && ok) {
        tc_fence_after();
        const DescParts a_tt = smem_desc_parts(sb + bl::TB, 16384, 1024, 2);
        const DescParts b_x = smem_desc_parts(sb + bl::XI, 16384, 1024, 2);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            umma_bf16_p(tmem + 320 + L16, a_tt.lo + mnmaj(kk), a_tt.hi, b_x.lo + mnmaj(kk), b_x.hi,
                        idesc_g(64, 64, true, true), kk > 0);
        umma_commit(bar_mma);
    }
    ok = mma_done(ok);
    // ---- dA = -tril_-1(Y) -> DA image ----
    if (ok && warp < 4) {
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2) {
            float x[32];
            tmem_ld32(tmem + lane_base + 320 + 32 * c2, x);
            tmem_wait_ld();
            if (hi) {
#pragma unroll
                for (int j = 0; j < 32; ++j) x[j] = (32 * c2 + j < row) ? -x[j] : 0.f;
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    *reinterpret_cast<uint4 *>(sm + bl::DA + img_off(row, 32 * c2 + 8 * e, 8192)) = pack8(x + 8 * e, 1.f);
            }
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    // ---- phase 2d: D_bV = T^T dV_new; D_bKg = T^T dW + dA Kinv; D_Kinv += dA^T bKg ----
    if (tid == 0 && ok) {
        tc_fence_after();
        const DescParts a_tt = smem_desc_parts(sb + bl::TB, 16384, 1024, 2);
        const DescParts b_dvn = smem_desc_parts(sb + bl::DVN, 8192, 1024, 2);
        const DescParts b_dw = smem_desc_parts(sb + bl::DW, 8192, 1024, 2);
        const DescParts a_da = smem_desc_parts(sb + bl::DA, 16, 1024, 2);
        const DescParts a_dat = smem_desc_parts(sb + bl::DA, 16384, 1024, 2);
        const DescParts b_kinv = smem_desc_parts(sb + bl::KI, 8192, 1024, 2);
        const DescParts b_bkg = smem_desc_parts(sb + bl::KQ, 16384, 1024, 2);
        constexpr uint32_t IMM = idesc_g(64, 128, true, true), IKM = idesc_g(64, 128, false, true);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            umma_bf16_p(tmem + 384, a_tt.lo + mnmaj(kk), a_tt.hi, b_dvn.lo + mnmaj(kk), b_dvn.hi, IMM, kk > 0);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            umma_bf16_p(tmem + 384 + L16, a_tt.lo + mnmaj(kk), a_tt.hi, b_dw.lo + mnmaj(kk), b_dw.hi, IMM, kk > 0);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            umma_bf16_p(tmem + 384 + L16, a_da.lo + kmaj(kk, 8192), a_da.hi, b_kinv.lo + mnmaj(kk), b_kinv.hi, IKM, 1);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            umma_bf16_p(tmem + 128 + L16, a_dat.lo + mnmaj(kk), a_dat.hi, b_bkg.lo + mnmaj(kk), b_bkg.hi, IMM, 1);
        umma_commit(bar_mma);
    }
    ok = mma_done(ok);

    // ---- finale: per token row and 32-channel group ----
    if (tid == 0 && ok) ok = mbar_wait(bar_fin, 0);
    ok = __syncthreads_and(ok);
    float *dG = reinterpret_cast<float *>(sm + bl::KQ);        // [64][128] fp32 (bKg, Qg are dead)
    if (ok) {
        // warp: token rows 16 sub .. 16 sub + 15 (one per lane of each half),
        // 64 of the channels (csel), 16 per step; lane half hi takes 8 of
        // each step's 16.  Lane hi = 0 holds the +0 tile (Q, Kt, bV) of all
        // 16 channels, lane hi = 1 the +16 tile (Kinv, bKg); three shuffles
        // per channel pair give each half the other tile's values of its own
        // channels.
        const int csel = warp >> 2;
        const int i = row;
        const bool live = i < len;
        const float br = bet[i];
        float dbp = 0.f;
#pragma unroll 1
        for (int step = 0; step < 4; ++step) {
            const int cc = 2 * (step >> 1) + csel;
            const int ch0 = 32 * cc + 16 * (step & 1);      // this step's 16 channels
            const int cm = ch0 + 8 * hi;                     // this lane's 8
            float a[16], b[16], c[16];
            tmem_ld16(tmem + lane_base + ch0, a);            // D_Q | (dead D_W)
            tmem_ld16(tmem + lane_base + 128 + ch0, b);      // D_Kt | D_Kinv
            tmem_ld16(tmem + lane_base + 384 + ch0, c);      // D_bV | D_bKg
            tmem_wait_ld();
            float dQg[8], dKt[8], dbV[8], dKinv[8], dbKg[8];
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
                const float s1 = __shfl_xor_sync(0xffffffffu, hi ? b[jj] : a[8 + jj], 16);
                const float s2 = __shfl_xor_sync(0xffffffffu, hi ? c[jj] : b[8 + jj], 16);
                const float s3 = __shfl_xor_sync(0xffffffffu, c[8 + jj], 16);
                dQg[jj] = hi ? s1 : a[jj];
                dKt[jj] = hi ? s2 : b[jj];
                dbV[jj] = hi ? s3 : c[jj];
                dKinv[jj] = hi ? b[8 + jj] : s1;
                dbKg[jj] = hi ? c[8 + jj] : s2;
            }
            const uint32_t so = (cm >> 6) * 8192 + sw(i, cm & 63);
            const uint4 qx = *reinterpret_cast<const uint4 *>(sm + bl::DO + so);
            const uint4 kx = *reinterpret_cast<const uint4 *>(sm + bl::VN + so);
            const uint4 vx = *reinterpret_cast<const uint4 *>(sm + bl::V + so);
            const uint32_t qw[4] = {qx.x, qx.y, qx.z, qx.w}, kw[4] = {kx.x, kx.y, kx.z, kx.w},
                           vw[4] = {vx.x, vx.y, vx.z, vx.w};
            float oq[8], ok_[8], ov[8], ktv[8];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float2 qf = bf16x2_to_float2(qw[u]), kf = bf16x2_to_float2(kw[u]),
                             vf = bf16x2_to_float2(vw[u]);
                const float qs[2] = {qf.x, qf.y}, ks[2] = {kf.x, kf.y}, vs[2] = {vf.x, vf.y};
#pragma unroll
                for (int w2 = 0; w2 < 2; ++w2) {
                    const int jj = 2 * u + w2, ch = cm + jj;
                    const float g2 = G2[gsw(i, ch)], gc2 = G2[gsw(63, ch)];
                    const float eg = ex2_approx(g2), em = ex2_approx(-g2), egc = ex2_approx(gc2);
                    const float kt = ks[w2] * em * egc;
                    oq[jj] = dQg[jj] * eg;
                    ok_[jj] = dbKg[jj] * br * eg + (dKinv[jj] + dKt[jj] * egc) * em;
                    ov[jj] = dbV[jj] * br;
                    if (live) dbp = fmaf(dbKg[jj] * ks[w2], eg, fmaf(dbV[jj], vs[w2], dbp));
                    dG[gsw(i, ch)] = live ? dQg[jj] * qs[w2] * eg + dbKg[jj] * br * ks[w2] * eg -
                                                dKinv[jj] * ks[w2] * em - dKt[jj] * kt
                                          : 0.f;
                    ktv[jj] = live ? dKt[jj] * kt : 0.f;
                }
            }
            if (live) {
                const size_t grow = ((size_t)(t0 + i) * H + h) * D + cm;
                if (v8) {
                    // 8 channels = one 32-byte sector per gradient and row
                    st_v8(dq + grow, oq);
                    st_v8(dk + grow, ok_);
                    st_v8(dv + grow, ov);
                } else {
                    float4 *pq = reinterpret_cast<float4 *>(dq + grow);
                    float4 *pk = reinterpret_cast<float4 *>(dk + grow);
                    float4 *pv = reinterpret_cast<float4 *>(dv + grow);
                    pq[0] = make_float4(oq[0], oq[1], oq[2], oq[3]); pq[1] = make_float4(oq[4], oq[5], oq[6], oq[7]);
                    pk[0] = make_float4(ok_[0], ok_[1], ok_[2], ok_[3]); pk[1] = make_float4(ok_[4], ok_[5], ok_[6], ok_[7]);
                    pv[0] = make_float4(ov[0], ov[1], ov[2], ov[3]); pv[1] = make_float4(ov[4], ov[5], ov[6], ov[7]);
                }
            }
            // column sums over the half's 16 token rows (xor steps stay inside
            // each half), one slot per channel and row group (no atomics)
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
                float t = ktv[jj];
                t += __shfl_xor_sync(0xffffffffu, t, 1);
                t += __shfl_xor_sync(0xffffffffu, t, 2);
                t += __shfl_xor_sync(0xffffffffu, t, 4);
                t += __shfl_xor_sync(0xffffffffu, t, 8);
                if (l16 == 0) kts[(warp & 3) * 128 + cm + jj] = t;
            }
        }
        // dbeta of the row: both halves' channels, both channel groups (csel)
        dbp += __shfl_xor_sync(0xffffffffu, dbp, 16);
        if (hi == 0 && live) dbs[csel * 64 + i] = dbp;
    }
    __syncthreads();
    // dg = reverse cumsum of dG inside the chunk, the G_C terms on the last
    // row: two threads per channel, rows 32-63 (hf = 1) and 0-31 (hf = 0),
    // each scanning its 32 rows in registers; the lower half then adds the
    // upper half's total, passed through shared memory
    if (ok) {
        const int c = tid & 127, hf = tid >> 7;
        const int r0 = 32 * hf;
        float x[32];
#pragma unroll
        for (int t = 0; t < 32; ++t) x[t] = dG[gsw(r0 + t, c)];
        if (hf) x[31] += (kts[c] + kts[128 + c]) + (kts[256 + c] + kts[384 + c]) +
                         degc[c] * ex2_approx(G2[gsw(63, c)]);
#pragma unroll
        for (int t = 30; t >= 0; --t) x[t] += x[t + 1];
        __syncthreads();                         // every thread has read kts
        if (hf) kts[c] = x[0];
        __syncthreads();
        const float up = hf ? 0.f : kts[c];
#pragma unroll
        for (int t = 0; t < 32; ++t)
            if (r0 + t < len) dg[((size_t)(t0 + r0 + t) * H + h) * D + c] = x[t] + up;
        if (tid < len) dbeta[(size_t)(t0 + tid) * H + h] = dbs[tid] + dbs[64 + tid];
    }
    if (!ok && tid == 0) {
        if (!bad) set_device_error(err, kErrWaitTimeout);
        // never leave with copies in flight into this CTA's shared memory
        mbar_wait(bar_g, 0, 1u << 20);
        mbar_wait(bar_ld, 0, 1u << 20);
        mbar_wait(bar_in2, 0, 1u << 20);
        if (in3_issued) mbar_wait(bar_in3, 0, 1u << 20);
        if (fin_issued) mbar_wait(bar_fin, 0, 1u << 20);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace

cudaError_t launch_chunk_bwd_local(const void *q, const void *k, const void *v, const float *g,
                                   const float *beta, const void *dout, const int32_t *cu,
                                   const int32_t *coff, int N, int T, int total_T, int H,
                                   int max_chunks, const unsigned char *s_img,
                                   const unsigned char *v_img, const unsigned char *dsp_img,
                                   const unsigned char *dvn_img, float *dq, float *dk, float *dv,
                                   float *dg, float *dbeta, int *err, cudaStream_t st)
{
    CUtensorMap mq, mk, mv, mg, mdo;
    cudaError_t e = make_token_map(&mq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, H, total_T, 64, CU_TENSOR_MAP_SWIZZLE_128B);
    if (e == cudaSuccess) e = make_token_map(&mk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, H, total_T, 64, CU_TENSOR_MAP_SWIZZLE_128B);
    if (e == cudaSuccess) e = make_token_map(&mv, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, H, total_T, 64, CU_TENSOR_MAP_SWIZZLE_128B);
    if (e == cudaSuccess) e = make_token_map(&mg, g, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, H, total_T, D, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (e == cudaSuccess) e = make_token_map(&mdo, dout, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, H, total_T, 64, CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess) return e;
    const size_t smem = bl::BYTES + 1024;
    e = cudaFuncSetAttribute(chunk_bwd_local_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(max_chunks, H);
    chunk_bwd_local_kernel<<<grid, NT, smem, st>>>(
        mq, mk, mv, mg, mdo, (const __nv_bfloat16 *)q, (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)v, beta,
        cu, coff, N, T, total_T, H, (T + C - 1) / C, s_img, v_img, dsp_img, dvn_img, dq, dk, dv, dg, dbeta,
        (((uintptr_t)dq | (uintptr_t)dk | (uintptr_t)dv) & 31u) == 0, err);
    return cudaGetLastError();
}

}  // namespace kda

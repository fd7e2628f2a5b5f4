// decode_chunk_tc.cu -- the L-token KDA decode on a slot-indexed state pool in
// the chunk form, one 64-token chunk at a time on tcgen05 tensor cores (bf16
// operands, fp32 accumulation in tensor memory, fp32 state), dk = dv = 128.
//
// Kimi Linear paper notes (paper-notes-site): section 2 gives the recurrence,
// section 3 the chunkwise form: the chunk's writes gathered by a WY-like
// representation (W, U), then one product with the fixed-size state.  For
// chunk j of one (sequence, head), with G the chunk-local inclusive cumsum of
// g and S the state entering the chunk:
//     A_ij = beta_i sum_c k_ic k_jc e^{G_ic - G_jc}  (j < i)
//     P_ij =        sum_c q_ic k_jc e^{G_ic - G_jc}  (j <= i)
//     T = (I + A)^-1,  W = T (beta K e^G),  U = T (beta V)
//     V_new = U - W S,   O = (Q e^G) S + P V_new
//     S <- Diag(e^{G_C}) S + (K e^{G_C - G})^T V_new
// The prefill's algebra (chunk_prep.cu, chunk_chain_tc.cu) with the state read
// from and written back to the pool inside the same CTA, so nothing but the
// inputs, the outputs and the state crosses HBM.  One CTA per (sequence,
// head) item at a time, persistent (two per SM), each 64-token chunk:
//
//   forms, MMA-AP  [beta K e^G ; Q e^G] (K e^{-G})^T (M = 128)  -> A, P
//   T (fp32, diagonal substitution and tf32 block levels), bf16
//   MMA-W / MMA-U  T (beta K e^G) -> W, T (beta V) -> U           (M = 64 each)
//   state pass     -W (bf16); S (bf16, MN-major B operand);
//                  e^{G_C} S (fp32) into TMEM by tcgen05.st
//   MMA-S          U + (-W) S -> V_new in place, (Q e^G) S          (M = 64 each)
//   MMA-O          P V_new accumulated onto (Q e^G) S -> O          (M = 64)
//   MMA-upd        (K e^{G_C - G})^T V_new accumulated onto e^{G_C} S -> S'   (M = 128)
//   epilogue       O (bf16); S' leaves TMEM at the top of the next unit
//
// TMEM (256 columns): columns 0-127 hold two M = 64 accumulators, one on
// lanes 0-15 of each 32-lane sub-partition (+0: W, then (Q e^G) S and O),
// one on lanes 16-31 (+16: U, then V_new); columns 128-255 hold the state
// (e^{G_C} S, then S').  K e^{G_C - G} leaves the forms pass from registers
// into a per-CTA slot of global scratch (it stays in L2) and returns by TMA
// when shared memory is free again.  The next chunk's inputs are staged by
// TMA into regions of the current chunk that are dead: g, q and k once MMA-S
// has read -W, Q e^G and S, v once MMA-O and MMA-upd have read V_new.
//
// A chunk whose decay leaves the chunk-start exponent range (every e^{+-G}
// and e^{G_C - G} within e^{+-80}) is not computed here: its (item, first
// token) goes to a list, the item's later chunks are skipped, and
// decode_chunk_kernel finishes the listed items from that token on (16-token
// blocks with exact exponentials), so any finite g <= 0 is accepted.
#include <cudaTypedefs.h>

#include <algorithm>

#include "chunk_ws.h"
#include "common.cuh"
#include "kernels.h"
#include "prep_common.cuh"
#include "sm100.cuh"

namespace kda {
using namespace prep;
namespace {
namespace dtc {
// Tiles are K-major with the 128-byte swizzle (rows of 64 bf16 = 128 bytes,
// 16-byte chunk j of row r at j ^ (r % 8), 8-row groups 1024 bytes apart).
constexpr int OFF_KQ = 0;        // per 64-channel block b at b * 16384: [k rows | q rows]
                                 //   k -> beta k e^G -> W,  q -> q e^G
constexpr int OFF_G = 32768;     // g (fp32 [64][128], TMA) until the cumsum has read it
constexpr int OFF_KI = 32768;    // k e^{-G} (block b at b * 8192), then A (fp32 64 x 64)
constexpr int OFF_Z = 49152;     // diagonal blocks of A and form_T scratch, then T (bf16)
constexpr int OFF_S = 32768;     // S (bf16): value atom a at a * 16384, [128 channel rows][64 values]
constexpr int OFF_V = 65536;     // v -> beta v -> V_new (value atom a at a * 8192, [64 token rows][64])
constexpr int OFF_TB = 81920;    // P (bf16, 64 swizzled rows), read by MMA-O
constexpr int OFF_TM = 90112;    // T (fp32 64 x 64), then K e^{G_C - G} ([128 channel rows][64 tokens])
constexpr int OFF_GS = 106496;   // per-sub-chunk sums of g [4][128]
constexpr int OFF_EGC = OFF_GS + 4 * D * 4;   // e^{G_C} [128]
constexpr int OFF_BETA = OFF_EGC + D * 4;     // beta [64]
constexpr int OFF_BAR = OFF_BETA + C * 4;     // mbarriers: g, q, kv, mma, kt
constexpr int OFF_TSLOT = OFF_BAR + 5 * 8;    // TMEM base address
constexpr int OFF_UNIT = OFF_TSLOT + 8;       // the next unit (one thread writes it)
constexpr int BYTES = OFF_UNIT + 16;
constexpr uint32_t TX_G = C * D * 4;
constexpr uint32_t TX_Q = 2 * 8192;
constexpr uint32_t TX_KV = 4 * 8192;
constexpr uint32_t TMEM_COLS = 256;
constexpr uint32_t KT_BYTES = 16384;
constexpr float RANGE2 = 80.f * 1.4426950408889634f;   // e^{+-80} bound, in log2 units
static_assert(OFF_TM % 1024 == 0 && OFF_TB % 1024 == 0 && OFF_V % 1024 == 0 && OFF_Z % 1024 == 0 &&
              OFF_BAR % 8 == 0 && BYTES + 1024 <= 113 * 1024, "layout: two CTAs per SM");
enum { B_G = 0, B_Q, B_KV, B_MMA, B_KT };
// byte offset of (row r, channel c in 0..63) in a swizzled 64-channel block
__device__ __forceinline__ int sw(int r, int c) {
    return r * 128 + ((((c >> 3) ^ (r & 7))) << 4) + ((c & 7) << 1);
}
}  // namespace dtc

// 32 lanes x 32 columns of 32-bit from registers: thread i of the warp
// writes lane (base + i)
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n" ::"r"(taddr),
        "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
        "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
        "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
        "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
        "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
        "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
        "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
        "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
        "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
        "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
        "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
        : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory"); }

// 256-bit global accesses (32-byte aligned addresses): a warp's row-per-
// thread pattern then moves whole 32-byte sectors, half the instructions
__device__ __forceinline__ void ld_v8(const float *p, float *v) {
    asm volatile("ld.global.v8.f32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];\n"
                 : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7])
                 : "l"(p));
}
__device__ __forceinline__ void st_v8(float *p, const float *v) {
    asm volatile("st.global.v8.f32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};\n" ::"l"(p), "f"(v[0]), "f"(v[1]), "f"(v[2]),
                 "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7])
                 : "memory");
}
__device__ __forceinline__ void st_v8_bf16(void *p, const float *v) {
    asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};\n" ::"l"(p), "r"(pack_bf16(v[0], v[1])),
                 "r"(pack_bf16(v[2], v[3])), "r"(pack_bf16(v[4], v[5])), "r"(pack_bf16(v[6], v[7])),
                 "r"(pack_bf16(v[8], v[9])), "r"(pack_bf16(v[10], v[11])), "r"(pack_bf16(v[12], v[13])),
                 "r"(pack_bf16(v[14], v[15]))
                 : "memory");
}

// 16 lanes x 32 columns, twice: threads 0-15 read lanes base .. base + 15 at
// columns [c, c + 32), threads 16-31 the same lanes at [c + 32, c + 64)
__device__ __forceinline__ void tmem_ld16x2(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.16x32bx2.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32], 32;\n"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// one chunk of one item: item it = n * H + h, chunk index c (-1 = none)
struct Unit { int it, c; };

__global__ void __launch_bounds__(NT, 2)
decode_chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                       const float *__restrict__ beta, float *__restrict__ pool,
                       const int32_t *__restrict__ slots, int num_slots, __nv_bfloat16 *__restrict__ out,
                       const __grid_constant__ CUtensorMap tm_kt,
                       int N, int H, int L, unsigned char *__restrict__ kt_scratch,
                       int2 *__restrict__ fb_list, int *__restrict__ fb_count, int *__restrict__ err)
{
    using namespace sm100;
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + dtc::OFF_BAR);
    uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + dtc::OFF_TSLOT);
    Unit *uslot = reinterpret_cast<Unit *>(sm + dtc::OFF_UNIT);
    float *gs = reinterpret_cast<float *>(sm + dtc::OFF_GS);
    float *egc_s = reinterpret_cast<float *>(sm + dtc::OFF_EGC);
    float *bet = reinterpret_cast<float *>(sm + dtc::OFF_BETA);
    unsigned char *kts = kt_scratch + (size_t)blockIdx.x * dtc::KT_BYTES;
    const int items = N * H;
    const int nch = (L + C - 1) / C;
    const uint32_t sb = smem_u32(sm);

    // The next item at or after `it` (grid stride) whose slot is valid; -1 if
    // none (thread 0 only).
    auto next_valid = [&](int it) -> int {
        for (; it < items; it += gridDim.x) {
            const int n = it / H;
            const int s = slots ? slots[n] : n;
            if (s >= 0 && s < num_slots) return it;
            set_device_error(err, kErrBadSlot);
        }
        return -1;
    };
    auto state_of = [&](int it) -> float * {
        const int n = it / H, h = it - n * H;
        const int s = slots ? slots[n] : n;
        return pool + ((size_t)s * H + h) * (size_t)(D * D);
    };
    // token rows [row0, row0 + len) of the unit in the [N * L, H, 128] views
    auto row0 = [&](const Unit &u) { return (u.it / H) * L + C * u.c; };
    auto len_of = [&](const Unit &u) { return min(C, L - C * u.c); };

    // barrier bookkeeping (thread 0): armed-and-unwaited mask and the parity
    // each barrier completes next
    uint32_t pend = 0, par = 0;
    auto arm = [&](int b) { pend |= 1u << b; };
    auto wait_bar = [&](int b) -> bool {
        const bool ok = mbar_wait(bars + b, (par >> b) & 1u);
        if (ok) { pend &= ~(1u << b); par ^= 1u << b; }
        return ok;
    };
    // g, q and k of unit u (thread 0); v follows on the same barrier as k.
    // The first chunk of an item also asks L2 for the item's state.
    auto load_gqk = [&](const Unit &u, const float *S_first) {
        const int h = u.it % H, r = row0(u);
        mbar_arrive_expect_tx(bars + dtc::B_G, dtc::TX_G);
        tma_load_3d(sm + dtc::OFF_G, &tm_g, 0, h, r, bars + dtc::B_G);
        arm(dtc::B_G);
        mbar_arrive_expect_tx(bars + dtc::B_Q, dtc::TX_Q);
        mbar_arrive_expect_tx(bars + dtc::B_KV, dtc::TX_KV);
#pragma unroll
        for (int b = 0; b < 2; ++b) {
            tma_load_3d(sm + dtc::OFF_KQ + b * 16384 + 8192, &tm_q, 64 * b, h, r, bars + dtc::B_Q);
            tma_load_3d(sm + dtc::OFF_KQ + b * 16384, &tm_k, 64 * b, h, r, bars + dtc::B_KV);
        }
        arm(dtc::B_Q);
        arm(dtc::B_KV);
        if (S_first) {
#pragma unroll
            for (int p = 0; p < 4; ++p) bulk_prefetch_l2(S_first + p * 4096, 16384);
        }
    };
    auto load_v = [&](const Unit &u) {
        const int h = u.it % H, r = row0(u);
#pragma unroll
        for (int b = 0; b < 2; ++b)
            tma_load_3d(sm + dtc::OFF_V + b * 8192, &tm_v, 64 * b, h, r, bars + dtc::B_KV);
    };
    auto load_beta = [&](const Unit &u) {
        float bt = 0.f;
        if (tid < len_of(u)) bt = beta[(size_t)(row0(u) + tid) * H + u.it % H];
        return bt;
    };
    auto next_unit = [&](const Unit &u, bool skip_item) -> Unit {
        if (!skip_item && u.c + 1 < nch) return Unit{u.it, u.c + 1};
        const int it = next_valid(u.it + gridDim.x);
        return Unit{it, it < 0 ? -1 : 0};
    };

    if (tid == 0) {
        for (int b = 0; b < 5; ++b) mbar_init(bars + b, 1);
        fence_mbar_init();
        const int it = next_valid(blockIdx.x);
        const Unit u{it, it < 0 ? -1 : 0};
        *uslot = u;
        if (it >= 0) { load_gqk(u, state_of(it)); load_v(u); }
    }
    if (warp == 0) { tmem_alloc(tslot, dtc::TMEM_COLS); tmem_relinquish(); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tslot;
    float bt_cur = 0.f;
    Unit cur = *uslot;
    if (tid < C && cur.it >= 0) bt_cur = load_beta(cur);
    bool ok = true;
    const int qd = warp & 3, hf = warp >> 2;            // TMEM lane quarter, 64-column half
    const uint32_t lanes = (uint32_t)(qd * 32) << 16;
    // The new state of a unit stays in TMEM columns 128-255 until the top of
    // the next unit, where it goes to the pool while that unit's inputs land
    // (its state pass writes those columns again).  Row c = TMEM lane.
    float *S_out = nullptr;
    auto store_state = [&](float *Sg) {
        float *srow = Sg + (qd * 32 + lane) * D + 64 * hf;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            float x[32];
            tmem_ld32(tmem + lanes + 128u + 64u * hf + 32u * half, x);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 4; ++j) st_v8(srow + 32 * half + 8 * j, x + 8 * j);
        }
    };

    while (cur.it >= 0) {
    if (S_out) { store_state(S_out); S_out = nullptr; }
    const int h = cur.it % H, len = len_of(cur), t0 = row0(cur);
    float *S = state_of(cur.it);
    // the unit after this one, and its state if it starts an item (thread 0):
    // the next item's slot is loaded now and used while MMA-W/U runs
    Unit nx{-1, -1};
    const float *nxS = nullptr;
    const int nit = cur.it + gridDim.x;
    int nslot = -1;
    if (tid == 0 && cur.c + 1 >= nch && nit < items) nslot = slots ? slots[nit / H] : nit / H;
    if (tid < C) bet[tid] = bt_cur;
    if (tid == 0) ok = wait_bar(dtc::B_G);
    ok = __syncthreads_and(ok);
    if (!ok) break;

    // ---- g: thread (sub-chunk I, channels c0, c0 + 1); local cumsum ----
    const int I = tid >> 6, c0 = 2 * (tid & 63);
    const int cb = c0 >> 6, cc = c0 & 63;
    float2 G[16];
    {
        const float *gsm = reinterpret_cast<const float *>(sm + dtc::OFF_G);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int r = 16 * I + i;
            G[i] = make_float2(0.f, 0.f);
            if (r < len) G[i] = *reinterpret_cast<const float2 *>(gsm + r * D + c0);
        }
    }
    constexpr float L2E = 1.4426950408889634f;
    G[0].x *= L2E; G[0].y *= L2E;
#pragma unroll
    for (int i = 1; i < 16; ++i) { G[i].x = fmaf(G[i].x, L2E, G[i - 1].x); G[i].y = fmaf(G[i].y, L2E, G[i - 1].y); }
    *reinterpret_cast<float2 *>(gs + I * D + c0) = G[15];
    __syncthreads();
    float2 GC = make_float2(0.f, 0.f), PF = make_float2(0.f, 0.f);
#pragma unroll
    for (int J = 0; J < 4; ++J) {
        const float2 sj = *reinterpret_cast<const float2 *>(gs + J * D + c0);
        if (J < I) { PF.x += sj.x; PF.y += sj.y; }
        GC.x += sj.x; GC.y += sj.y;
    }
    bool bad = false;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        G[i].x += PF.x; G[i].y += PF.y;
        bad |= !(fabsf(G[i].x) <= dtc::RANGE2 && fabsf(G[i].y) <= dtc::RANGE2 &&
                 GC.x - G[i].x <= dtc::RANGE2 && GC.y - G[i].y <= dtc::RANGE2);
    }
    if (tid == 0) ok = wait_bar(dtc::B_Q) && wait_bar(dtc::B_KV);
    ok = __syncthreads_and(ok);
    if (!ok) break;
    if (__syncthreads_or(bad)) {
        // out of the chunk-start range: the item goes to the list from this
        // chunk on, and the next item's first chunk is staged at once
        fence_proxy_async_smem();
        __syncthreads();
        if (tid == 0) {
            const int idx = atomicAdd(fb_count, 1);
            fb_list[idx] = make_int2(cur.it, C * cur.c);
            const Unit nx = next_unit(cur, true);
            *uslot = nx;
            if (nx.it >= 0) { load_gqk(nx, state_of(nx.it)); load_v(nx); }
        }
        __syncthreads();
        cur = *uslot;
        if (tid < C && cur.it >= 0) bt_cur = load_beta(cur);
        continue;
    }

    // ---- decayed forms: q e^G, beta k e^G, beta v (in place), k e^{-G}
    // (over the consumed g); K e^{G_C - G} to the scratch slot; e^{G_C} ----
    {
        const float2 egc = make_float2(ex2_approx(GC.x), ex2_approx(GC.y));
        if (I == 0) *reinterpret_cast<float2 *>(egc_s + c0) = make_float2(exp2f(GC.x), exp2f(GC.y));
        uint32_t kt[2][8];
        float2 kt_prev = make_float2(0.f, 0.f);
        unsigned char *kq = sm + dtc::OFF_KQ + cb * 16384;
        unsigned char *ki = sm + dtc::OFF_KI + cb * 8192;
        unsigned char *vv = sm + dtc::OFF_V + cb * 8192;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int r = 16 * I + i;
            const int o = dtc::sw(r, cc);
            const float2 eg = make_float2(ex2_approx(G[i].x), ex2_approx(G[i].y));
            const float2 em = make_float2(ex2_approx(-G[i].x), ex2_approx(-G[i].y));
            float2 qf = bf16x2_to_float2(*reinterpret_cast<const uint32_t *>(kq + 8192 + o));
            float2 kf = bf16x2_to_float2(*reinterpret_cast<const uint32_t *>(kq + o));
            float2 vf = bf16x2_to_float2(*reinterpret_cast<const uint32_t *>(vv + o));
            if (r >= len) { qf = kf = vf = make_float2(0.f, 0.f); }
            const float br = bet[r];
            const float2 b2 = make_float2(br, br);
            const float2 kinv = __fmul2_rn(kf, em);
            const float2 kt2 = __fmul2_rn(kinv, egc);
            *reinterpret_cast<uint32_t *>(kq + 8192 + o) = pack_bf16x2(__fmul2_rn(qf, eg));
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
        // plain rows of 64 tokens (128 bytes): tokens 16 I .. 16 I + 15 of
        // channels c0, c0 + 1 are one 32-byte piece each
#pragma unroll
        for (int e = 0; e < 2; ++e)
            asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};\n" ::"l"(kts + (c0 + e) * 128 + 32 * I),
                         "r"(kt[e][0]), "r"(kt[e][1]), "r"(kt[e][2]), "r"(kt[e][3]), "r"(kt[e][4]), "r"(kt[e][5]),
                         "r"(kt[e][6]), "r"(kt[e][7])
                         : "memory");
        // the slot returns by TMA (async proxy), swizzled for MMA-upd
        asm volatile("fence.proxy.async.global;\n" ::: "memory");
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();

    if (tid == 0) {
        tc_fence_after();
        // A: [beta k e^G ; q e^G] K-major (M = 128), B: k e^{-G} K-major (N = 64)
        constexpr uint32_t ID_AP = idesc_bf16(128, 64, false);
        const DescParts da = smem_desc_parts(sb + dtc::OFF_KQ, 16, 1024, 2);
        const DescParts db = smem_desc_parts(sb + dtc::OFF_KI, 16, 1024, 2);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
            umma_bf16_p(tmem, da.lo + (((kk >> 2) * 16384 + (kk & 3) * 32) >> 4), da.hi,
                        db.lo + (((kk >> 2) * 8192 + (kk & 3) * 32) >> 4), db.hi, ID_AP, kk > 0);
        umma_commit(bars + dtc::B_MMA);
        arm(dtc::B_MMA);
        ok = wait_bar(dtc::B_MMA);
    }
    ok = __syncthreads_and(ok);
    tc_fence_after();
    if (!ok) break;

    // ---- A (masked j < i) -> fp32 for form_T; P (masked j <= i) -> image ----
    float *Am = reinterpret_cast<float *>(sm + dtc::OFF_KI);
    float *Tm = reinterpret_cast<float *>(sm + dtc::OFF_TM);
    float *Ad = reinterpret_cast<float *>(sm + dtc::OFF_Z);
    if (warp < 4) {
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
            unsigned char *img = sm + dtc::OFF_TB;
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
    form_T_padded_diag(Am, Ad, Tm, reinterpret_cast<float *>(sm + dtc::OFF_Z), tid);
    // T -> bf16 over the substitution scratch, one swizzled 128-byte row per token row i
    {
        const int i = tid >> 2, jq = tid & 3;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int jg = 2 * jq + hh;
            const float4 lo = *reinterpret_cast<const float4 *>(Tm + i * 64 + 4 * ((2 * jg) ^ (i & 7)));
            const float4 hi = *reinterpret_cast<const float4 *>(Tm + i * 64 + 4 * ((2 * jg + 1) ^ (i & 7)));
            *reinterpret_cast<uint4 *>(sm + dtc::OFF_Z + i * 128 + ((jg ^ (i & 7)) << 4)) =
                make_uint4(pack_bf16(lo.x, lo.y), pack_bf16(lo.z, lo.w), pack_bf16(hi.x, hi.y),
                           pack_bf16(hi.z, hi.w));
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    // M = 64 products share TMEM columns 0-127: one accumulator on lanes 0-15
    // of each sub-partition (+0), one on lanes 16-31 (+16); warp lane l reads
    // row 16 (warp % 4) + (l % 16) of the +0 tile (l < 16) or the +16 tile
    constexpr uint32_t L16 = 16u << 16;
    constexpr uint32_t ID64 = idesc_bf16(64, 128, true);     // A K-major, B MN-major, 64 x 128
    constexpr uint32_t ID128 = idesc_bf16(128, 128, true);   // 128 x 128
    if (tid == 0) {
        tc_fence_after();
        // W = T (beta K e^G) -> +0, U = T (beta V) -> +16 (A: T K-major, K = 64
        // tokens; B: tokens along K, 64-channel atoms along N)
        const DescParts ta = smem_desc_parts(sb + dtc::OFF_Z, 16, 1024, 2);
        const DescParts bw = smem_desc_parts(sb + dtc::OFF_KQ, 16384, 1024, 2);
        const DescParts bu = smem_desc_parts(sb + dtc::OFF_V, 8192, 1024, 2);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            umma_bf16_p(tmem, ta.lo + ((kk * 32) >> 4), ta.hi, bw.lo + ((kk * 2048) >> 4), bw.hi, ID64, kk > 0);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            umma_bf16_p(tmem + L16, ta.lo + ((kk * 32) >> 4), ta.hi, bu.lo + ((kk * 2048) >> 4), bu.hi, ID64,
                        kk > 0);
        umma_commit(bars + dtc::B_MMA);
        arm(dtc::B_MMA);
        // K e^{G_C - G} back from the slot over T (fp32), read above
        mbar_arrive_expect_tx(bars + dtc::B_KT, dtc::KT_BYTES);
        tma_load_3d(sm + dtc::OFF_TM, &tm_kt, 0, 0, blockIdx.x, bars + dtc::B_KT);
        arm(dtc::B_KT);
        if (cur.c + 1 < nch) {
            nx = Unit{cur.it, cur.c + 1};
        } else if (nslot >= 0 && nslot < num_slots) {
            nx = Unit{nit, 0};
            nxS = pool + ((size_t)nslot * H + nit % H) * (size_t)(D * D);
        } else {
            nx = next_unit(cur, false);
            if (nx.it >= 0) nxS = state_of(nx.it);
        }
        ok = wait_bar(dtc::B_MMA);
    }
    ok = __syncthreads_and(ok);
    tc_fence_after();
    if (!ok) break;

    {
        // -W (rows 16 qd + l, l < 16, of the +0 tile) as bf16 over the dead k
        // rows: the A operand that turns U into V_new = U - W S in place
        const int r = 16 * qd + (lane & 15), half = lane >> 4;
        unsigned char *dst = sm + dtc::OFF_KQ + hf * 16384 + r * 128;
        {
            float x[32];
            tmem_ld16x2(tmem + lanes + 64u * hf, x);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int jc = 4 * half + j;
                const float *w = x + 8 * j;
                *reinterpret_cast<uint4 *>(dst + ((jc ^ (r & 7)) << 4)) =
                    make_uint4(pack_bf16(-w[0], -w[1]), pack_bf16(-w[2], -w[3]),
                               pack_bf16(-w[4], -w[5]), pack_bf16(-w[6], -w[7]));
            }
        }
        // S row c = TMEM lane, values 64 hf .. + 63: bf16 into the MN-major B
        // operand of MMA-S (value atom hf, [128 channel rows][64 values]), and
        // e^{G_C}[c] S[c][v] in fp32 into TMEM columns 128-255, where MMA-upd
        // accumulates the rank-64 update onto it
        const int c = qd * 32 + lane;
        const float gc = egc_s[c];
        const float *srow = S + c * D + 64 * hf;
        unsigned char *brow = sm + dtc::OFF_S + hf * 16384 + c * 128;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            float so[32];
#pragma unroll
            for (int j = 0; j < 4; ++j) ld_v8(srow + 32 * half + 8 * j, so + 8 * j);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float *a = so + 8 * j;
                const int jc = 4 * half + j;
                *reinterpret_cast<uint4 *>(brow + ((jc ^ (c & 7)) << 4)) =
                    make_uint4(pack_bf16(a[0], a[1]), pack_bf16(a[2], a[3]), pack_bf16(a[4], a[5]),
                               pack_bf16(a[6], a[7]));
            }
#pragma unroll
            for (int j = 0; j < 32; ++j) so[j] *= gc;
            tmem_st32(tmem + lanes + 128u + 64u * hf + 32u * half, *reinterpret_cast<const float (*)[32]>(so));
        }
        tmem_wait_st();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
        tc_fence_after();
        // V_new = U + (-W) S onto +16, Q e^G S -> +0 (A: K-major, K = 128
        // channels in two atoms; B: S MN-major)
        const DescParts dw = smem_desc_parts(sb + dtc::OFF_KQ, 16, 1024, 2);
        const DescParts dq = smem_desc_parts(sb + dtc::OFF_KQ + 8192, 16, 1024, 2);
        const DescParts bs = smem_desc_parts(sb + dtc::OFF_S, 16384, 1024, 2);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
            umma_bf16_p(tmem + L16, dw.lo + (((kk >> 2) * 16384 + (kk & 3) * 32) >> 4), dw.hi,
                        bs.lo + ((kk * 2048) >> 4), bs.hi, ID64, 1u);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
            umma_bf16_p(tmem, dq.lo + (((kk >> 2) * 16384 + (kk & 3) * 32) >> 4), dq.hi,
                        bs.lo + ((kk * 2048) >> 4), bs.hi, ID64, kk > 0);
        umma_commit(bars + dtc::B_MMA);
        arm(dtc::B_MMA);
        ok = wait_bar(dtc::B_MMA);
    }
    ok = __syncthreads_and(ok);
    tc_fence_after();
    if (!ok) break;
    // k, q, g, W and S are read: the next unit's g, q and k go over them
    if (tid == 0) {
        *uslot = nx;
        if (nx.it >= 0) load_gqk(nx, nxS);
    }

    // ---- V_new (rows 16 qd + l - 16, l >= 16, of the +16 tile) -> bf16 over
    // beta v, as the MN-major B operand of MMA-O and MMA-upd ----
    {
        const int r = 16 * qd + (lane & 15), half = lane >> 4;
        unsigned char *dst = sm + dtc::OFF_V + hf * 8192 + r * 128;
        {
            float x[32];
            tmem_ld16x2(tmem + lanes + L16 + 64u * hf, x);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int jc = 4 * half + j;
                const float *a = x + 8 * j;
                *reinterpret_cast<uint4 *>(dst + ((jc ^ (r & 7)) << 4)) =
                    make_uint4(pack_bf16(a[0], a[1]), pack_bf16(a[2], a[3]), pack_bf16(a[4], a[5]),
                               pack_bf16(a[6], a[7]));
            }
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    float bt_next = 0.f;
    {
        const Unit nb = *uslot;    // written by thread 0 before the barrier above
        if (tid < C && nb.it >= 0) bt_next = load_beta(nb);
    }
    if (tid == 0) {
        tc_fence_after();
        ok = wait_bar(dtc::B_KT);
        if (ok) {
            // O = Q e^G S + P V_new onto +0 (A: P K-major, K = 64 tokens);
            // S' = e^{G_C} S + (K e^{G_C - G})^T V_new onto columns 128-255
            // (A: [128 channel rows][64 tokens] K-major)
            const DescParts tp = smem_desc_parts(sb + dtc::OFF_TB, 16, 1024, 2);
            const DescParts tk = smem_desc_parts(sb + dtc::OFF_TM, 16, 1024, 2);
            const DescParts bv = smem_desc_parts(sb + dtc::OFF_V, 8192, 1024, 2);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                umma_bf16_p(tmem, tp.lo + ((kk * 32) >> 4), tp.hi, bv.lo + ((kk * 2048) >> 4), bv.hi, ID64, 1u);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                umma_bf16_p(tmem + 128, tk.lo + ((kk * 32) >> 4), tk.hi, bv.lo + ((kk * 2048) >> 4), bv.hi,
                            ID128, 1u);
            umma_commit(bars + dtc::B_MMA);
            arm(dtc::B_MMA);
            ok = wait_bar(dtc::B_MMA);
        }
    }
    ok = __syncthreads_and(ok);
    tc_fence_after();
    if (!ok) break;
    // V_new, P and K e^{G_C - G} are read: the next unit's v goes over V_new
    if (tid == 0 && nx.it >= 0) load_v(nx);

    // ---- epilogue: O (rows of the +0 tile, l < 16); the new state leaves at
    // the top of the next unit ----
    {
        const int r = 16 * qd + (lane & 15), half = lane >> 4;
        {
            float x[32];
            tmem_ld16x2(tmem + lanes + 64u * hf, x);
            tmem_wait_ld();
            if (r < len) {
                __nv_bfloat16 *dst = out + ((size_t)(t0 + r) * H + h) * D + 64 * hf + 32 * half;
                st_v8_bf16(dst, x);
                st_v8_bf16(dst + 16, x + 16);
            }
        }
    }
    S_out = S;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    cur = *uslot;
    bt_cur = bt_next;
    }   // units

    if (ok && S_out) store_state(S_out);
    if (!ok && tid == 0) {
        // a bounded wait ran out: report it, and let what this CTA has in
        // flight (loads, copies, MMAs) finish, with bounded waits again,
        // before its shared and tensor memory are released
        set_device_error(err, kErrWaitTimeout);
        for (int b = 0; b < 5; ++b)
            if (pend & (1u << b)) mbar_wait(bars + b, (par >> b) & 1u);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, dtc::TMEM_COLS);
}

}  // namespace

size_t decode_chunk_tc_scratch_bytes(int N, int H, int sms) {
    const size_t slots = (size_t)2 * sms * dtc::KT_BYTES;
    const size_t list = ((size_t)N * H * sizeof(int2) + 255) & ~(size_t)255;
    return slots + list + 256;
}

cudaError_t launch_decode_chunk_tc(const void *q, const void *k, const void *v, const float *g,
                                   const float *beta, float *pool, const int32_t *slots, int num_slots,
                                   void *out, int N, int H, int L, int sms, void *scratch, int *err,
                                   cudaStream_t st)
{
    if (N == 0 || L == 0) return cudaSuccess;
    if ((long long)N * L > 0x7fffffffLL) return cudaErrorInvalidValue;
    const int items = N * H;
    const int grid = std::min(items, 2 * sms);
    unsigned char *kt_scratch = static_cast<unsigned char *>(scratch);
    int2 *list = reinterpret_cast<int2 *>(kt_scratch + (size_t)2 * sms * dtc::KT_BYTES);
    int *count = reinterpret_cast<int *>(reinterpret_cast<unsigned char *>(list) +
                                         (((size_t)items * sizeof(int2) + 255) & ~(size_t)255));
    cudaError_t e = cudaMemsetAsync(count, 0, sizeof(int), st);
    if (e != cudaSuccess) return e;
    CUtensorMap mq, mk, mv, mg;
    const int rows = N * L;
    e = make_token_map(&mq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, H, rows, 64, CU_TENSOR_MAP_SWIZZLE_128B);
    if (e == cudaSuccess)
        e = make_token_map(&mk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, H, rows, 64, CU_TENSOR_MAP_SWIZZLE_128B);
    if (e == cudaSuccess)
        e = make_token_map(&mv, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, H, rows, 64, CU_TENSOR_MAP_SWIZZLE_128B);
    if (e == cudaSuccess)
        e = make_token_map(&mg, g, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, H, rows, D, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (e != cudaSuccess) return e;
    // the K e^{G_C - G} slots: [grid][128 channel rows][64 tokens] bf16, one
    // box per slot, 128-byte swizzle on arrival
    CUtensorMap mkt;
    {
        PFN_cuTensorMapEncodeTiled_v12000 fn = tensor_map_encoder();
        if (!fn) return cudaErrorNotSupported;
        const cuuint64_t dims[3] = {64, 128, (cuuint64_t)grid};
        const cuuint64_t strides[2] = {128, dtc::KT_BYTES};
        const cuuint32_t box[3] = {64, 128, 1};
        const cuuint32_t estr[3] = {1, 1, 1};
        if (fn(&mkt, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, kt_scratch, dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    const size_t smem = dtc::BYTES + 1024;
    e = cudaFuncSetAttribute(decode_chunk_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    decode_chunk_tc_kernel<<<grid, NT, smem, st>>>(mq, mk, mv, mg, beta, pool, slots, num_slots,
                                                   (__nv_bfloat16 *)out, mkt, N, H, L, kt_scratch, list,
                                                   count, err);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    // the listed items, from their first out-of-range chunk on
    return launch_decode_chunk_list(q, k, v, g, beta, pool, slots, num_slots, out, N, H, L, list, count,
                                    err, st);
}

}  // namespace kda

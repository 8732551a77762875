// Tensor-core (tcgen05 + TMA) split-KV verification attention for bf16 caches.
//
// Serves sd_verify_attention when the GQA group times the new rows, R = G * n_q, is between
// 16 and 128 (7B-like layers verify gamma+1 = 6..9 rows with G = 7: R = 42..63).
//
// One CTA per (split, KV head g, sequence b); 6 warps, one CTA per SM:
//   warps 0-3  softmax: TMEM lane r holds query row r (rows ordered (i, h), h fastest; rows
//              R..127 are padding and never read back)
//   warp 4     TMA producer: K and V tiles of 128 positions (128-byte swizzle) into a
//              3-4 stage shared-memory ring (a stage's K is released once S is computed, its V
//              once P.V is) (contiguous caches: one 4-D box per half of
//              head_dim; paged caches: one box per 16-position page)
//   warp 5     MMA issuer (one elected thread) and TMEM owner
// Per tile t (double-buffered S in TMEM):
//   S_t = Q K_t^T        tcgen05.mma kind::f16, M=128, N=128, A = Q (smem, K-major),
//                        B = K tile (smem, K-major), fp32 accumulators in TMEM
//   softmax              each thread reads its row of S_t from TMEM, applies the causal
//                        mask j <= kv_len - n_q + i, updates its running max (base 2) and
//                        writes P_t = 2^(s - m) as bf16 over S_t in TMEM.  The running max
//                        used for the exponent only moves when the true max grows by more
//                        than 2^8 ("lazy rescale"), so O is rarely touched.
//   O += P_t V_t         tcgen05.mma with A = P_t from TMEM, B = V tile (smem, MN-major)
// Partial outputs (O, max, sum) go to the split workspace exactly like the CUDA-core engine,
// or, with a single split, O / sum is written directly.
// Every wait on an mbarrier is bounded (1 s); on expiry the CTA records SD_DEVERR_TIMEOUT,
// drains its own copies and MMAs (again bounded), frees TMEM and exits.
#include <cuda.h>
#include <cuda_bf16.h>

#include "sd_internal.h"

namespace sd {
namespace {

constexpr int kTile = 128;            // positions per tile
constexpr int kRows = 128;            // MMA M
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kThreads = 6 * 32;
constexpr uint32_t kTmemCols = 512;   // S0 [0,128) S1 [128,256) O [256, 256+D)
constexpr uint32_t kColO = 256;
constexpr float kRescaleLog2 = 8.0f;
constexpr unsigned long long kWaitNs = 1000000000ull;
constexpr uint32_t kHalfBytes = kTile * 128;  // one 64-column half of a 128-row tile

template <int D>
struct Cfg {
    static constexpr int kHalves = D / 64;
    static constexpr int kTileBytes = kTile * D * 2;
    static constexpr int kStages = D == 128 ? 3 : 4;
    static constexpr int kQBytes = kRows * D * 2;
    static constexpr int kBarOffset = kQBytes + kStages * 2 * kTileBytes;
    static constexpr int kSmem = kBarOffset + 256 + 1024;  // barriers (<= 4S+8 words) + slack
};

// ---------------------------------------------------------------- PTX wrappers ------------

__device__ __forceinline__ uint32_t saddr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ unsigned long long now_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Bounded wait for the phase of `bar` with the given parity.  Returns false when the CTA is
// aborting (this wait timed out, or another one did).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                          int32_t *dev_err) {
    if (mbar_try(bar, parity)) return true;
    const unsigned long long t0 = now_ns();
    while (true) {
        if (mbar_try(bar, parity)) return true;
        if (*abort_flag) return false;
        if (now_ns() - t0 > kWaitNs) {
            *abort_flag = 1;
            set_dev_err(dev_err, SD_DEVERR_TIMEOUT);
            return false;
        }
    }
}

__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap *map, uint32_t bar,
                                            int x, int y, int z, int w) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "r"(z), "r"(w)
        : "memory");
}

__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tc_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// K-major operand, 128-byte swizzle: rows of 128 bytes, 8-row atoms 1024 bytes apart.
__device__ __forceinline__ uint64_t desc_k_sw128(uint32_t addr) {
    return (uint64_t)((addr & 0x3FFFFu) >> 4) | (1ull << 16) | (64ull << 32) | (1ull << 46) |
           (2ull << 61);
}

// MN-major operand, 128-byte swizzle: 64 MN-elements per 128-byte row, K rows 128 bytes
// apart, 8-row atoms 1024 bytes apart (SBO), 64-element MN groups lbo bytes apart.
__device__ __forceinline__ uint64_t desc_mn_sw128(uint32_t addr, uint32_t lbo) {
    return (uint64_t)((addr & 0x3FFFFu) >> 4) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           (64ull << 32) | (1ull << 46) | (2ull << 61);
}

// kind::f16 instruction descriptor: fp32 accumulate, bf16 A and B, M = 128.
__host__ __device__ constexpr uint32_t idesc_bf16(int n, bool b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) |
           ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kRows >> 4) << 24);
}

__device__ __forceinline__ void mma_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                       uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}

__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc,
                                       uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
        "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
        : "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane (load and wait in one statement, so
// no use of the values can be scheduled before the wait).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n\t"
        "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
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

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};\n\t"
        "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15])
        : "memory");
}

// All 128 fp32 columns [taddr, taddr+128) of this thread's TMEM lane, load + wait in one
// statement.
__device__ __forceinline__ void tmem_ld128(uint32_t taddr, float (&v)[128]) {
    uint32_t r[128];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x128.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,"
        "%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,"
        "%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63,%64,%65,%66,%67,"
        "%68,%69,%70,%71,%72,%73,%74,%75,%76,%77,%78,%79,%80,%81,%82,%83,%84,%85,%86,%87,%88,%89,"
        "%90,%91,%92,%93,%94,%95,%96,%97,%98,%99,%100,%101,%102,%103,%104,%105,%106,%107,%108,"
        "%109,%110,%111,%112,%113,%114,%115,%116,%117,%118,%119,%120,%121,%122,%123,%124,%125,"
        "%126,%127}, [%128];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]),
          "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]),
          "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]),
          "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]),
          "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]),
          "=r"(r[61]), "=r"(r[62]), "=r"(r[63]), "=r"(r[64]), "=r"(r[65]), "=r"(r[66]),
          "=r"(r[67]), "=r"(r[68]), "=r"(r[69]), "=r"(r[70]), "=r"(r[71]), "=r"(r[72]),
          "=r"(r[73]), "=r"(r[74]), "=r"(r[75]), "=r"(r[76]), "=r"(r[77]), "=r"(r[78]),
          "=r"(r[79]), "=r"(r[80]), "=r"(r[81]), "=r"(r[82]), "=r"(r[83]), "=r"(r[84]),
          "=r"(r[85]), "=r"(r[86]), "=r"(r[87]), "=r"(r[88]), "=r"(r[89]), "=r"(r[90]),
          "=r"(r[91]), "=r"(r[92]), "=r"(r[93]), "=r"(r[94]), "=r"(r[95]), "=r"(r[96]),
          "=r"(r[97]), "=r"(r[98]), "=r"(r[99]), "=r"(r[100]), "=r"(r[101]), "=r"(r[102]),
          "=r"(r[103]), "=r"(r[104]), "=r"(r[105]), "=r"(r[106]), "=r"(r[107]), "=r"(r[108]),
          "=r"(r[109]), "=r"(r[110]), "=r"(r[111]), "=r"(r[112]), "=r"(r[113]), "=r"(r[114]),
          "=r"(r[115]), "=r"(r[116]), "=r"(r[117]), "=r"(r[118]), "=r"(r[119]), "=r"(r[120]),
          "=r"(r[121]), "=r"(r[122]), "=r"(r[123]), "=r"(r[124]), "=r"(r[125]), "=r"(r[126]),
          "=r"(r[127])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 128; ++i) v[i] = __uint_as_float(r[i]);
}

// 64 packed columns to this thread's TMEM lane, store + wait in one statement.
__device__ __forceinline__ void tmem_st64(uint32_t taddr, const uint32_t (&r)[64]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x64.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,"
        "%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,"
        "%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63,%64};\n\t"
        "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
        "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
        "r"(r[29]), "r"(r[30]), "r"(r[31]), "r"(r[32]), "r"(r[33]), "r"(r[34]), "r"(r[35]),
        "r"(r[36]), "r"(r[37]), "r"(r[38]), "r"(r[39]), "r"(r[40]), "r"(r[41]), "r"(r[42]),
        "r"(r[43]), "r"(r[44]), "r"(r[45]), "r"(r[46]), "r"(r[47]), "r"(r[48]), "r"(r[49]),
        "r"(r[50]), "r"(r[51]), "r"(r[52]), "r"(r[53]), "r"(r[54]), "r"(r[55]), "r"(r[56]),
        "r"(r[57]), "r"(r[58]), "r"(r[59]), "r"(r[60]), "r"(r[61]), "r"(r[62]), "r"(r[63])
        : "memory");
}

__device__ __forceinline__ float max3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// 2^x with the hardware approximation (relative error ~2^-22; P is rounded to bf16 anyway).
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&p);
}

// ---------------------------------------------------------------- the kernel --------------

struct TcMaps {
    CUtensorMap k;
    CUtensorMap v;
};

template <int D, bool PAGED>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const AttnParams p, const __grid_constant__ TcMaps maps) {
    using C = Cfg<D>;
    constexpr int S = C::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = smem;
    uint8_t *sKV = smem + C::kQBytes;  // stage s: K at s*2*tile, V at s*2*tile + tile
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::kBarOffset);
    // barrier slots: k_full[S], v_full[S], k_empty[S], v_empty[S], s_full[2], p_full[2],
    // o_done, drain.  A stage's K half is released as soon as S = Q K^T is computed, its V
    // half once P.V is, so the next K copy starts a softmax earlier.
    const uint32_t bar0 = saddr(bars);
    auto BAR = [&](int i) { return bar0 + 8u * (uint32_t)i; };
    const int KF = 0, VF = S, KE = 2 * S, VE = 3 * S, SF = 4 * S, PF = 4 * S + 2, OD = 4 * S + 4,
              DR = 4 * S + 5;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 4 * S + 6);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int b = blockIdx.z, g = blockIdx.y, split = blockIdx.x;
    const KVView &kv = p.kv;
    const int G = p.group;
    const int q0 = __ldg(p.q_start + b);
    const int n_q = __ldg(p.q_start + b + 1) - q0;
    const int kv_len = __ldg(kv.kv_len + b);
    const int R = n_q * G;
    if (n_q < 1 || R > kRows || n_q > p.max_q_rows || q0 + n_q > p.rows_cap || kv_len < n_q ||
        (PAGED && kv_len > kv.max_pages * kPageSize)) {
        if (tid == 0 && n_q != 0) set_dev_err(p.dev_err, SD_DEVERR_SHAPE);
        return;
    }
    const int n_tiles = (kv_len + kTile - 1) / kTile;
    const int tile_lo = (int)((int64_t)n_tiles * split / p.n_splits);
    const int tile_hi = (int)((int64_t)n_tiles * (split + 1) / p.n_splits);
    const int n_my = tile_hi - tile_lo;
    const int n_active = (R + 31) / 32;  // softmax warps holding real rows

    if (warp == kMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         saddr(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(BAR(KF + s), 1);
            mbar_init(BAR(VF + s), 1);
            mbar_init(BAR(KE + s), 1);
            mbar_init(BAR(VE + s), 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(BAR(SF + s), 1);
            mbar_init(BAR(PF + s), 32 * n_active);
        }
        mbar_init(BAR(OD), 1);
        mbar_init(BAR(DR), 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // Q rows into shared memory in the 128-byte swizzled K-major layout (rows >= R are zero).
    if (warp < 4) {
        constexpr int CPR = D / 8;  // 16-byte chunks per row
        for (int e = tid; e < kRows * CPR; e += 128) {
            const int r = e / CPR, c = e % CPR;
            uint4 val = make_uint4(0, 0, 0, 0);
            if (r < R) {
                const int64_t off = ((int64_t)(q0 + r / G) * p.h_q + g * G + r % G) * D + c * 8;
                val = __ldg(reinterpret_cast<const uint4 *>(
                    reinterpret_cast<const unsigned short *>(p.q) + off));
            }
            const int half = c >> 3, cc = c & 7;
            *reinterpret_cast<uint4 *>(sQ + half * kHalfBytes + r * 128 + ((cc ^ (r & 7)) << 4)) =
                val;
        }
        fence_async_smem();
    }
    tc_before();
    __syncthreads();
    tc_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == kProducerWarp) {
        // ---------------------------------------------------------- TMA producer ----------
        if (lane == 0) {
            int pages[kTile / kPageSize];
            for (int t = 0; t < n_my; ++t) {
                const int s = t % S, use = t / S;
                const int p0 = (tile_lo + t) * kTile;
                const uint32_t dK = saddr(sKV + (size_t)s * 2 * C::kTileBytes);
                const uint32_t dV = dK + C::kTileBytes;
                if (PAGED) {
                    for (int pg = 0; pg < kTile / kPageSize; ++pg) {
                        const int pos = p0 + pg * kPageSize;
                        int page = kv.num_pages;  // out of range: zero-filled box
                        if (pos < kv_len) {
                            const int e = __ldg(kv.block_table + (int64_t)b * kv.max_pages +
                                                pos / kPageSize);
                            if (e >= 0 && e < kv.num_pages)
                                page = e;
                            else
                                set_dev_err(p.dev_err, SD_DEVERR_PAGE);
                        }
                        pages[pg] = page;
                    }
                }
                for (int half = 0; half < 2; ++half) {  // K, then V
                    const int full = half == 0 ? KF : VF, empty = half == 0 ? KE : VE;
                    const uint32_t dst = half == 0 ? dK : dV;
                    const CUtensorMap *map = half == 0 ? &maps.k : &maps.v;
                    if (t >= S && !mbar_wait(BAR(empty + s), (use - 1) & 1, abort_flag, p.dev_err))
                        break;
                    mbar_arrive_tx(BAR(full + s), C::kTileBytes);
                    if (!PAGED) {
#pragma unroll
                        for (int h = 0; h < C::kHalves; ++h)
                            tma_load_4d(dst + h * kHalfBytes, map, BAR(full + s), h * 64, p0, g, b);
                    } else {
                        for (int pg = 0; pg < kTile / kPageSize; ++pg)
#pragma unroll
                            for (int h = 0; h < C::kHalves; ++h)
                                tma_load_4d(dst + h * kHalfBytes + pg * kPageSize * 128, map,
                                            BAR(full + s), h * 64, 0, g, pages[pg]);
                    }
                }
                if (*abort_flag) break;
            }
        }
    } else if (warp == kMmaWarp) {
        // ---------------------------------------------------------- MMA issuer ------------
        // Lane 0 waits and issues; the decision is broadcast so the warp stays converged.
        // S = Q K^T of tile t+1 is issued before waiting for the softmax of tile t, so the
        // tensor core computes it while the softmax warps work.
        const uint32_t idesc_qk = idesc_bf16(kTile, false);
        const uint32_t idesc_pv = idesc_bf16(D, true);
        const uint32_t q_base = saddr(sQ);
        bool issued = false;
        auto issue_qk = [&](int t) -> bool {
            const int s = t % S, use = t / S, sb = t & 1;
            const uint32_t kb = saddr(sKV + (size_t)s * 2 * C::kTileBytes);
            bool ok = true;
            if (lane == 0) ok = mbar_wait(BAR(KF + s), use & 1, abort_flag, p.dev_err);
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok) return false;
            tc_after();
            if (lane == 0) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
                    mma_ss(tmem + sb * kTile, desc_k_sw128(q_base + off), desc_k_sw128(kb + off),
                           idesc_qk, kk > 0 ? 1u : 0u);
                }
                mma_commit(BAR(SF + sb));
                mma_commit(BAR(KE + s));
                issued = true;
            }
            __syncwarp();
            return true;
        };
        bool alive = n_my > 0 ? issue_qk(0) : true;
        for (int t = 0; alive && t < n_my; ++t) {
            const int s = t % S, use = t / S, sb = t & 1;
            if (t + 1 < n_my && !issue_qk(t + 1)) break;
            bool ok = true;
            if (lane == 0)
                ok = mbar_wait(BAR(PF + sb), (t >> 1) & 1, abort_flag, p.dev_err) &&
                     mbar_wait(BAR(VF + s), use & 1, abort_flag, p.dev_err);
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok) break;
            // V rows past the end of the sequence may hold anything (NaN included): zero
            // them so that 0 * V cannot poison O.
            uint8_t *vs = sKV + (size_t)s * 2 * C::kTileBytes + C::kTileBytes;
            const int valid = min(kTile, kv_len - (tile_lo + t) * kTile);
            if (valid < kTile) {
                const int nchunk = (kTile - valid) * 8;  // 16-byte chunks per half
                for (int h = 0; h < C::kHalves; ++h)
                    for (int e = lane; e < nchunk; e += 32)
                        *reinterpret_cast<uint4 *>(vs + h * kHalfBytes + valid * 128 + e * 16) =
                            make_uint4(0, 0, 0, 0);
                fence_async_smem();
                __syncwarp();
            }
            tc_after();
            if (lane == 0) {
                const uint32_t vb = saddr(vs);
#pragma unroll
                for (int kk = 0; kk < kTile / 16; ++kk)
                    mma_ts(tmem + kColO, tmem + sb * kTile + kk * 8,
                           desc_mn_sw128(vb + kk * 2048, kHalfBytes), idesc_pv,
                           (t > 0 || kk > 0) ? 1u : 0u);
                mma_commit(BAR(VE + s));
                mma_commit(BAR(OD));
            }
            __syncwarp();
        }
        // Drain: every MMA this warp issued has completed once the drain barrier flips.
        const bool any_issued = __any_sync(0xffffffffu, issued);
        if (lane == 0 && any_issued) {
            mma_commit(BAR(DR));
            const unsigned long long t0 = now_ns();
            while (!mbar_try(BAR(DR), 0) && now_ns() - t0 < kWaitNs) {
            }
        }
        __syncwarp();
    } else if (warp < n_active) {
        // ---------------------------------------------------------- softmax ---------------
        // tcgen05.ld / st are warp-collective: every lane executes them, row validity only
        // selects values, and decisions that gate them are made warp-uniform by votes.
        const unsigned FULL = 0xffffffffu;
        const int r = warp * 32 + lane;
        const bool row_ok = r < R;
        const int limit = kv_len - n_q + (row_ok ? r / G : 0);
        const int warp_limit = kv_len - n_q + (warp * 32) / G;  // smallest limit in this warp
        const float sl2 = p.scale_log2;
        const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
        float m_used = -INFINITY, l = 0.f;
        bool ok_run = true;
        for (int t = 0; t < n_my; ++t) {
            const int sb = t & 1;
            const int p0 = (tile_lo + t) * kTile;
            const bool got = mbar_wait(BAR(SF + sb), (t >> 1) & 1, abort_flag, p.dev_err);
            if (!__all_sync(FULL, got)) {
                ok_run = false;
                break;
            }
            tc_after();
            const uint32_t s_addr = lane_base + sb * kTile;
            float v[kTile];
            tmem_ld128(s_addr, v);
            // Interior tiles (every position visible to every row of this warp) skip masking.
            const bool interior = p0 + kTile - 1 <= warp_limit;
            float mx = -INFINITY;
            if (!interior) {
#pragma unroll
                for (int e = 0; e < kTile; ++e)
                    if (!(row_ok && p0 + e <= limit)) v[e] = -INFINITY;
            }
#pragma unroll
            for (int e = 0; e < kTile; e += 2) mx = max3(mx, v[e], v[e + 1]);
            mx = mx == -INFINITY ? -INFINITY : mx * sl2;
            const bool grow = mx > m_used + kRescaleLog2;
            const bool rescale_o = grow && m_used != -INFINITY;
            if (__any_sync(FULL, rescale_o)) {
                // O holds tiles < t: wait for the P.V of tile t-1, then rescale O in TMEM.
                // S_t was committed after the P.V of tile t-2 and the P.V of tile t needs this
                // warp's arrival, so o_done is in phase t-1 or t: its parity test is exact.
                const bool done = mbar_wait(BAR(OD), (t - 1) & 1, abort_flag, p.dev_err);
                if (!__all_sync(FULL, done)) {
                    ok_run = false;
                    break;
                }
                tc_after();
                const float corr = rescale_o ? ex2(m_used - mx) : 1.f;
                float o[32];
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    tmem_ld32(lane_base + kColO + c * 32, o);
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] *= corr;
                    tmem_st32(lane_base + kColO + c * 32, o);
                }
                l *= corr;
            }
            if (grow) m_used = mx;
            // P = 2^(s*scale - m).  Masked entries are -inf and give exactly 0; while no
            // position of the row has been visible (m = -inf) every entry is masked.
            const float neg_m = m_used == -INFINITY ? 0.f : -m_used;
            const float2 sc2 = make_float2(sl2, sl2), nm2 = make_float2(neg_m, neg_m);
            float2 acc2 = make_float2(0.f, 0.f);
            uint32_t pk[kTile / 2];
#pragma unroll
            for (int e = 0; e < kTile; e += 2) {
                const float2 x = __ffma2_rn(make_float2(v[e], v[e + 1]), sc2, nm2);
                const float2 pe = make_float2(ex2(x.x), ex2(x.y));
                acc2 = __fadd2_rn(acc2, pe);
                pk[e >> 1] = pack_bf16(pe.x, pe.y);
            }
            tmem_st64(s_addr, pk);
            const float sum = acc2.x + acc2.y;
            l += sum;
            tc_before();
            mbar_arrive(BAR(PF + sb));
        }
        // ---- epilogue ----
        // Wait on the one-shot drain barrier (committed after the last P.V), not on the
        // per-tile o_done barrier: here only the P.V of tiles < n_my - 2 is known to be
        // complete, so o_done could be two phases behind and its parity test would pass early.
        bool done = ok_run;
        if (ok_run && n_my > 0) done = mbar_wait(BAR(DR), 0, abort_flag, p.dev_err);
        const bool read_o = __all_sync(FULL, done) && n_my > 0;
        tc_after();
        const bool have = read_o && m_used != -INFINITY;
        const int i = row_ok ? r / G : 0, h = g * G + (row_ok ? r % G : 0);
        const int row = q0 + i;
        const float inv = (have && l > 0.f) ? 1.f / l : 0.f;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
            float o[32];
            if (read_o) {
                tmem_ld32(lane_base + kColO + c * 32, o);
            }
#pragma unroll
            for (int e = 0; e < 32; ++e)
                if (!have) o[e] = 0.f;
            if (!row_ok) continue;
            if (p.n_splits == 1) {
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 32; e += 2) pk[e >> 1] = pack_bf16(o[e] * inv, o[e + 1] * inv);
                uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<unsigned short *>(p.out) +
                                                       ((int64_t)row * p.h_q + h) * D + c * 32);
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
            } else {
                const int64_t base = ((int64_t)split * p.rows_cap + row) * p.h_q + h;
                float4 *dst = reinterpret_cast<float4 *>(p.ws_o + base * D + c * 32);
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    dst[e] = make_float4(o[4 * e], o[4 * e + 1], o[4 * e + 2], o[4 * e + 3]);
                if (c == 0) {
                    p.ws_ml[base * 2] = have ? m_used : -INFINITY;
                    p.ws_ml[base * 2 + 1] = have ? l : 0.f;
                }
            }
        }
    }

    // ---- teardown: the producer drains its own copies if the CTA aborted ----
    if (warp == kProducerWarp && lane == 0 && *abort_flag) {
        const unsigned long long t0 = now_ns();
        for (int t = (n_my > S ? n_my - S : 0); t < n_my; ++t) {
            const int s = t % S, use = t / S;
            while ((!mbar_try(BAR(KF + s), use & 1) || !mbar_try(BAR(VF + s), use & 1)) &&
                   now_ns() - t0 < kWaitNs) {
            }
        }
    }
    tc_before();
    __syncthreads();
    tc_after();
    if (warp == kMmaWarp)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(kTmemCols)
                     : "memory");
}

// ---------------------------------------------------------------- host side ---------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encoder() {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
        else
            cudaGetLastError();
    }
    return fn;
}

bool encode_maps(const AttnParams &p, int max_kv_len, TcMaps *maps) {
    EncodeTiledFn enc = encoder();
    if (!enc) return false;
    const KVView &kv = p.kv;
    const cuuint64_t d = (cuuint64_t)kv.head_dim;
    cuuint64_t dims[4], strides[3];
    cuuint32_t box[4] = {64, 0, 1, 1}, elem[4] = {1, 1, 1, 1};
    if (kv.page_size == 0) {
        cuuint64_t lcap;
        if (kv.h_kv > 1)
            lcap = (cuuint64_t)kv.stride_h / d;
        else if (p.batch > 1)
            lcap = (cuuint64_t)kv.stride_b / d;
        else
            lcap = (cuuint64_t)max_kv_len;
        if (lcap < (cuuint64_t)max_kv_len || lcap < 1) return false;
        dims[0] = d;
        dims[1] = lcap;
        dims[2] = (cuuint64_t)kv.h_kv;
        dims[3] = (cuuint64_t)p.batch;
        strides[0] = d * 2;
        strides[1] = (cuuint64_t)kv.stride_h * 2;
        strides[2] = (cuuint64_t)kv.stride_b * 2;
        if (kv.h_kv == 1) strides[1] = lcap * d * 2;
        if (p.batch == 1) strides[2] = strides[1] * (cuuint64_t)kv.h_kv;
        box[1] = kTile;
    } else {
        dims[0] = d;
        dims[1] = kPageSize;
        dims[2] = (cuuint64_t)kv.h_kv;
        dims[3] = (cuuint64_t)kv.num_pages;
        strides[0] = d * 2;
        strides[1] = (cuuint64_t)kPageSize * d * 2;
        strides[2] = (cuuint64_t)kv.h_kv * kPageSize * d * 2;
        box[1] = kPageSize;
    }
    for (int i = 0; i < 3; ++i)
        if (strides[i] % 16 != 0) return false;
    CUresult rk = enc(&maps->k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(kv.k), dims,
                      strides, box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    CUresult rv = enc(&maps->v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(kv.v), dims,
                      strides, box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return rk == CUDA_SUCCESS && rv == CUDA_SUCCESS;
}

template <int D, bool PAGED>
cudaError_t launch_t(const AttnParams &p, const AttnPlan &plan, const TcMaps &maps,
                     cudaStream_t s) {
    auto kern = attn_tc_kernel<D, PAGED>;
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             Cfg<D>::kSmem);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    dim3 grid(p.n_splits, p.kv.h_kv, p.batch);
    kern<<<grid, kThreads, Cfg<D>::kSmem, s>>>(p, maps);
    return cudaGetLastError();
}

}  // namespace

bool tc_supported(int kind, int dtype, int head_dim, int rows) {
    return kind == SD_ATTN_VERIFY && dtype == SD_BF16 && (head_dim == 64 || head_dim == 128) &&
           rows >= 16 && rows <= kRows;
}

cudaError_t launch_attention_tc(const AttnParams &p, const AttnPlan &plan, cudaStream_t s) {
    TcMaps maps;
    if (!encode_maps(p, plan.max_kv_len, &maps)) return cudaErrorNotSupported;
    const bool paged = p.kv.page_size != 0;
    if (p.kv.head_dim == 128)
        return paged ? launch_t<128, true>(p, plan, maps, s) : launch_t<128, false>(p, plan, maps, s);
    return paged ? launch_t<64, true>(p, plan, maps, s) : launch_t<64, false>(p, plan, maps, s);
}

}  // namespace sd

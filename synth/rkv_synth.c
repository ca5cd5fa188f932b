/*
 * Seeded synthetic KV caches for the residual KV-cache compression path.
 *
 * This module generates inputs only; it holds none of the compression
 * arithmetic.  Both the CUDA path and the CPU oracle are fed from the bits
 * it writes.
 *
 * Model of a cache (one (layer, sequence, kv-head) unit):
 *   - P key prototypes and P value prototypes, each ~N(0,1)^D;
 *   - token i draws a prototype id uniformly from {0..P-1} (same id for K and V);
 *   - K_i = Kproto[id] + sigma * N(0,1)^D,  V_i = Vproto[id] + sigma * N(0,1)^D;
 *   - optionally n_outlier distinct key channels per unit whose whole column
 *     (prototype + noise) is multiplied by outlier_scale.
 * Prototypes are global over the sequence, so the nearest earlier tokens of a
 * token lie anywhere in the context, which is the long-range similarity the
 * ResidualKV / DeltaKV pages report (p1 "Key Empirical Observations").
 *
 * Random numbers are counter based: every value is a pure function of
 * (seed, stream ids, counter), so any row of any unit can be regenerated on
 * its own.  The counter hash is the splitmix64 output function (Steele, Lea
 * and Flood, "Fast splittable pseudorandom number generators", OOPSLA 2014);
 * Gaussians come from the Box-Muller transform in double precision.
 * Values are rounded double -> float (round to nearest even) and, for bf16
 * outputs, float -> bf16 (round to nearest even).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define SYN_DTYPE_BF16 0
#define SYN_DTYPE_F32 1

enum {
    ROLE_KPROTO = 1,
    ROLE_VPROTO = 2,
    ROLE_ASSIGN = 3,
    ROLE_KNOISE = 4,
    ROLE_VNOISE = 5,
    ROLE_OUTLIER = 6,
    ROLE_QUERY = 7,
    ROLE_LENGTH = 8,
};

static const uint64_t GOLDEN = 0x9e3779b97f4a7c15ULL;

static inline uint64_t mix64(uint64_t z)
{
    z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ULL;
    z = (z ^ (z >> 27)) * 0x94d049bb133111ebULL;
    return z ^ (z >> 31);
}

static inline uint64_t derive(uint64_t s, uint64_t id) { return mix64(s + GOLDEN * (id + 1)); }

static inline uint64_t draw(uint64_t stream, uint64_t ctr) { return mix64(stream + GOLDEN * (ctr + 1)); }

/* uniform in (0, 1): 53 random bits, centred in their cell */
static inline double uniform01(uint64_t stream, uint64_t ctr)
{
    return ((double)(draw(stream, ctr) >> 11) + 0.5) * (1.0 / 9007199254740992.0);
}

/* standard normals 2m and 2m+1 of a stream (Box-Muller on uniform pair m) */
static inline void normal_pair(uint64_t stream, uint64_t m, double* z0, double* z1)
{
    const double u1 = uniform01(stream, 2 * m);
    const double u2 = uniform01(stream, 2 * m + 1);
    const double r = sqrt(-2.0 * log(u1));
    const double th = 6.283185307179586476925286766559 * u2;
    *z0 = r * cos(th);
    *z1 = r * sin(th);
}

/* standard normal number n of a stream */
static inline double normal(uint64_t stream, uint64_t n)
{
    double z0, z1;
    normal_pair(stream, n >> 1, &z0, &z1);
    return (n & 1) ? z1 : z0;
}

static inline uint16_t f32_to_bf16_rne(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7f800000u) == 0x7f800000u) /* inf / nan: truncate (nan kept quiet) */
        return (uint16_t)((u >> 16) | ((u & 0xffffu) ? 0x40u : 0u));
    const uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

static inline void store(void* out, int dtype, int64_t i, double v)
{
    const float f = (float)v;
    if (dtype == SYN_DTYPE_F32)
        ((float*)out)[i] = f;
    else
        ((uint16_t*)out)[i] = f32_to_bf16_rne(f);
}

typedef struct rkv_synth_params {
    uint64_t seed;        /* base seed */
    int32_t workload;     /* workload id, folded into every stream */
    int32_t head_dim;     /* D */
    int32_t n_proto;      /* P */
    int32_t n_outlier;    /* outlier key channels per unit (0 = none) */
    double sigma;         /* noise standard deviation */
    double outlier_scale; /* multiplier of the outlier key channels */
    int32_t dtype;        /* SYN_DTYPE_BF16 or SYN_DTYPE_F32 */
    int32_t pad_;
} rkv_synth_params;

static uint64_t unit_stream(const rkv_synth_params* p, int layer, int seq, int head, int role)
{
    uint64_t s = derive(p->seed, (uint64_t)(uint32_t)p->workload);
    s = derive(s, (uint64_t)(uint32_t)layer);
    s = derive(s, (uint64_t)(uint32_t)seq);
    s = derive(s, (uint64_t)(uint32_t)head);
    return derive(s, (uint64_t)role);
}

/* The outlier key channels of a unit: a partial Fisher-Yates shuffle of 0..D-1. */
int rkv_synth_outlier_channels(const rkv_synth_params* p, int layer, int seq, int head, int32_t* out)
{
    const int D = p->head_dim;
    int32_t perm[1024];
    if (D > 1024 || p->n_outlier > D)
        return -1;
    for (int c = 0; c < D; ++c)
        perm[c] = c;
    const uint64_t st = unit_stream(p, layer, seq, head, ROLE_OUTLIER);
    for (int i = 0; i < p->n_outlier; ++i) {
        const uint64_t r = draw(st, (uint64_t)i) >> 32;
        const int j = i + (int)((r * (uint64_t)(D - i)) >> 32);
        const int32_t t = perm[i];
        perm[i] = perm[j];
        perm[j] = t;
        out[i] = perm[i];
    }
    return p->n_outlier;
}

/* Prototype id of token t of a unit. */
int32_t rkv_synth_proto_id(const rkv_synth_params* p, int layer, int seq, int head, int64_t t)
{
    const uint64_t st = unit_stream(p, layer, seq, head, ROLE_ASSIGN);
    return (int32_t)(((draw(st, (uint64_t)t) >> 32) * (uint64_t)p->n_proto) >> 32);
}

/*
 * Rows [t0, t1) of one unit's K and V (row-major [t1-t0][D], element type
 * p->dtype).  Either output may be NULL.  scratch must hold 2*P*D doubles.
 */
int rkv_synth_kv(const rkv_synth_params* p, int layer, int seq, int head, int64_t t0, int64_t t1,
                 void* K_out, void* V_out, double* scratch)
{
    const int D = p->head_dim;
    const int P = p->n_proto;
    if (D <= 0 || (D & 1) || D > 1024 || P <= 0 || t1 < t0)
        return -1;
    double* kp = scratch;
    double* vp = scratch + (int64_t)P * D;
    const uint64_t s_kp = unit_stream(p, layer, seq, head, ROLE_KPROTO);
    const uint64_t s_vp = unit_stream(p, layer, seq, head, ROLE_VPROTO);
    for (int64_t i = 0; i < (int64_t)P * D; ++i) {
        kp[i] = normal(s_kp, (uint64_t)i);
        vp[i] = normal(s_vp, (uint64_t)i);
    }
    double kscale[1024];
    for (int c = 0; c < D; ++c)
        kscale[c] = 1.0;
    if (p->n_outlier > 0) {
        int32_t oc[1024];
        if (rkv_synth_outlier_channels(p, layer, seq, head, oc) < 0)
            return -1;
        for (int i = 0; i < p->n_outlier; ++i)
            kscale[oc[i]] = p->outlier_scale;
    }
    const uint64_t s_as = unit_stream(p, layer, seq, head, ROLE_ASSIGN);
    const uint64_t s_kn = unit_stream(p, layer, seq, head, ROLE_KNOISE);
    const uint64_t s_vn = unit_stream(p, layer, seq, head, ROLE_VNOISE);
    for (int64_t t = t0; t < t1; ++t) {
        const int64_t id = (int64_t)(((draw(s_as, (uint64_t)t) >> 32) * (uint64_t)P) >> 32);
        const int64_t row = (t - t0) * D;
        for (int c = 0; c < D; c += 2) { /* D is even: channel pairs share one Box-Muller pair */
            const uint64_t m = ((uint64_t)t * (uint64_t)D + (uint64_t)c) >> 1;
            double z0, z1;
            if (K_out) {
                normal_pair(s_kn, m, &z0, &z1);
                store(K_out, p->dtype, row + c, (kp[id * D + c] + p->sigma * z0) * kscale[c]);
                store(K_out, p->dtype, row + c + 1, (kp[id * D + c + 1] + p->sigma * z1) * kscale[c + 1]);
            }
            if (V_out) {
                normal_pair(s_vn, m, &z0, &z1);
                store(V_out, p->dtype, row + c, vp[id * D + c] + p->sigma * z0);
                store(V_out, p->dtype, row + c + 1, vp[id * D + c + 1] + p->sigma * z1);
            }
        }
    }
    return 0;
}

/* Decode queries q[B][Hq][D] = scale * N(0,1) for one (layer, step). */
int rkv_synth_query(const rkv_synth_params* p, int layer, int step, int B, int Hq, double scale, void* out)
{
    const int D = p->head_dim;
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < Hq; ++h) {
            uint64_t s = derive(p->seed, (uint64_t)(uint32_t)p->workload);
            s = derive(s, (uint64_t)(uint32_t)layer);
            s = derive(s, (uint64_t)(uint32_t)b);
            s = derive(s, (uint64_t)(uint32_t)h);
            s = derive(s, ROLE_QUERY);
            s = derive(s, (uint64_t)(uint32_t)step);
            for (int c = 0; c < D; ++c)
                store(out, p->dtype, ((int64_t)b * Hq + h) * D + c, scale * normal(s, (uint64_t)c));
        }
    return 0;
}

/* A sequence length uniform in [lo, hi]. */
int32_t rkv_synth_length(const rkv_synth_params* p, int seq, int32_t lo, int32_t hi)
{
    uint64_t s = derive(p->seed, (uint64_t)(uint32_t)p->workload);
    s = derive(s, ROLE_LENGTH);
    const uint64_t span = (uint64_t)(hi - lo) + 1;
    return lo + (int32_t)(((draw(s, (uint64_t)seq) >> 32) * span) >> 32);
}

/* FNV-1a over a byte buffer, for logging input checksums. */
uint64_t rkv_synth_checksum(const void* buf, int64_t nbytes, uint64_t h)
{
    const unsigned char* b = (const unsigned char*)buf;
    if (h == 0)
        h = 0xcbf29ce484222325ULL;
    for (int64_t i = 0; i < nbytes; ++i) {
        h ^= b[i];
        h *= 0x100000001b3ULL;
    }
    return h;
}

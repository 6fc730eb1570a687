// sbl_container.cpp -- the packed-layer container of include/sbl.h: a
// self-describing byte image of a packed layer (header, then the packed
// buffers), written and checked in host memory.  No device code and no
// CUDA calls: the caller moves the buffers between host and device.
#include <math.h>
#include <stdint.h>
#include <string.h>

#include "sbl.h"

namespace {

constexpr uint32_t kKnownFormats =
    SBL_FMT_PK2 | SBL_FMT_NM | SBL_FMT_I8 | SBL_FMT_BF16T | SBL_FMT_SP24 | SBL_FMT_T24;
constexpr size_t kAlign = 64;
const char kMagic[4] = {'S', 'B', 'L', 'P'};

// One stored buffer: which format bit it belongs to, which buffer of that
// format, and where its host pointer sits in sbl_host_buffers.
struct Slot {
    uint32_t format;
    sbl_buffer which;
    void *sbl_host_buffers::*member;
};

// The payload order of the layout comment in sbl.h.
const Slot kSlots[] = {
    {SBL_FMT_PK2, SBL_BUF_MAIN, &sbl_host_buffers::pk2},
    {SBL_FMT_NM, SBL_BUF_MAIN, &sbl_host_buffers::nm_values},
    {SBL_FMT_NM, SBL_BUF_NM_BITMAP, &sbl_host_buffers::nm_bitmap},
    {SBL_FMT_I8, SBL_BUF_MAIN, &sbl_host_buffers::i8},
    {SBL_FMT_BF16T, SBL_BUF_MAIN, &sbl_host_buffers::bf16t},
    {SBL_FMT_SP24, SBL_BUF_MAIN, &sbl_host_buffers::sp24_values},
    {SBL_FMT_SP24, SBL_BUF_SP24_META, &sbl_host_buffers::sp24_meta},
    {SBL_FMT_T24, SBL_BUF_MAIN, &sbl_host_buffers::t24_lo},
    {SBL_FMT_T24, SBL_BUF_T24_HI, &sbl_host_buffers::t24_hi},
};

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Bytes of one stored buffer (BF16T has in_features rows).
size_t slot_bytes(const sbl_layer_desc *d, const Slot &s)
{
    const size_t rows = static_cast<size_t>(s.format == SBL_FMT_BF16T ? d->in_features : d->out_features);
    return rows * sbl_packed_row_bytes(d, static_cast<sbl_format>(s.format), s.which);
}

// 0 when the mask is acceptable for the descriptor, else the status.
sbl_status check_formats(const sbl_layer_desc *d, uint32_t formats)
{
    if (formats & ~kKnownFormats) return SBL_ERR_INVALID_ARG;
    if ((formats & (SBL_FMT_SP24 | SBL_FMT_T24)) && d->n > 2) return SBL_ERR_UNSUPPORTED;
    return SBL_OK;
}

// Total image size for a valid descriptor and mask.
size_t image_bytes(const sbl_layer_desc *d, uint32_t formats)
{
    size_t off = SBL_CONTAINER_HEADER_BYTES;
    for (const Slot &s : kSlots)
        if (formats & s.format) off = round_up(off, kAlign) + slot_bytes(d, s);
    return off;
}

// 64-bit FNV-1a (offset basis 14695981039346656037, prime 1099511628211),
// continued from h over p[0 .. n).
uint64_t fnv1a64(uint64_t h, const uint8_t *p, size_t n)
{
    for (size_t i = 0; i < n; ++i) {
        h ^= p[i];
        h *= 1099511628211ull;
    }
    return h;
}

constexpr uint64_t kFnvBasis = 14695981039346656037ull;
constexpr size_t kHashAt = 40;  // the 8 hash bytes: the only bytes the hash skips

// The hash of an image of `total` bytes: every byte except bytes 40-47.
uint64_t image_hash(const uint8_t *img, size_t total)
{
    uint64_t h = fnv1a64(kFnvBasis, img, kHashAt);
    return fnv1a64(h, img + kHashAt + 8, total - kHashAt - 8);
}

void put32(uint8_t *p, uint32_t v)
{
    for (int i = 0; i < 4; ++i) p[i] = static_cast<uint8_t>(v >> (8 * i));
}

void put64(uint8_t *p, uint64_t v)
{
    for (int i = 0; i < 8; ++i) p[i] = static_cast<uint8_t>(v >> (8 * i));
}

uint32_t get32(const uint8_t *p)
{
    uint32_t v = 0;
    for (int i = 0; i < 4; ++i) v |= static_cast<uint32_t>(p[i]) << (8 * i);
    return v;
}

uint64_t get64(const uint8_t *p)
{
    uint64_t v = 0;
    for (int i = 0; i < 8; ++i) v |= static_cast<uint64_t>(p[i]) << (8 * i);
    return v;
}

int32_t as_i32(uint32_t v)
{
    int32_t r;
    memcpy(&r, &v, 4);
    return r;
}

uint32_t as_u32(int32_t v)
{
    uint32_t r;
    memcpy(&r, &v, 4);
    return r;
}

// Header and payload checks shared by sbl_container_info and _read.
sbl_status parse(const void *src, size_t src_bytes, sbl_layer_desc *desc, uint32_t *formats, float *gamma)
{
    if (!src || src_bytes < SBL_CONTAINER_HEADER_BYTES) return SBL_ERR_INVALID_ARG;
    const uint8_t *h = static_cast<const uint8_t *>(src);
    if (memcmp(h, kMagic, 4) != 0) return SBL_ERR_INVALID_ARG;
    if (get32(h + 4) != SBL_CONTAINER_VERSION) return SBL_ERR_UNSUPPORTED;
    sbl_layer_desc d;
    d.out_features = as_i32(get32(h + 8));
    d.in_features = as_i32(get32(h + 12));
    d.n = as_i32(get32(h + 16));
    d.m = as_i32(get32(h + 20));
    const uint32_t f = get32(h + 24);
    if (sbl_packed_row_bytes(&d, SBL_FMT_I8, SBL_BUF_MAIN) == 0) return SBL_ERR_SHAPE;
    const sbl_status st = check_formats(&d, f);
    if (st != SBL_OK) return SBL_ERR_INVALID_ARG;  // a writer never stores such a mask
    const uint64_t payload = get64(h + 32);
    const size_t expect = image_bytes(&d, f);
    if (payload != expect - SBL_CONTAINER_HEADER_BYTES || src_bytes < expect) return SBL_ERR_INVALID_ARG;
    for (int i = 52; i < SBL_CONTAINER_HEADER_BYTES; ++i)
        if (h[i] != 0) return SBL_ERR_INVALID_ARG;
    if (image_hash(h, expect) != get64(h + kHashAt)) return SBL_ERR_INVALID_ARG;
    if (desc) *desc = d;
    if (formats) *formats = f;
    if (gamma) {
        const uint32_t gb = get32(h + 28);
        memcpy(gamma, &gb, 4);
    }
    return SBL_OK;
}

}  // namespace

extern "C" {

size_t sbl_container_bytes(const sbl_layer_desc *desc, uint32_t formats)
{
    if (!desc || sbl_packed_row_bytes(desc, SBL_FMT_I8, SBL_BUF_MAIN) == 0) return 0;
    if (check_formats(desc, formats) != SBL_OK) return 0;
    return image_bytes(desc, formats);
}

sbl_status sbl_container_write(const sbl_layer_desc *desc, uint32_t formats, float gamma,
                               const sbl_host_buffers *src, void *dst, size_t dst_bytes)
{
    if (!desc || !src || !dst) return SBL_ERR_INVALID_ARG;
    if (sbl_packed_row_bytes(desc, SBL_FMT_I8, SBL_BUF_MAIN) == 0) return SBL_ERR_SHAPE;
    sbl_status st = check_formats(desc, formats);
    if (st != SBL_OK) return st;
    if (!isfinite(gamma)) return SBL_ERR_INVALID_ARG;
    for (const Slot &s : kSlots)
        if ((formats & s.format) && !(src->*s.member)) return SBL_ERR_INVALID_ARG;
    const size_t total = image_bytes(desc, formats);
    if (dst_bytes < total) return SBL_ERR_SHAPE;

    uint8_t *out = static_cast<uint8_t *>(dst);
    memset(out, 0, total);
    size_t off = SBL_CONTAINER_HEADER_BYTES;
    for (const Slot &s : kSlots) {
        if (!(formats & s.format)) continue;
        off = round_up(off, kAlign);
        const size_t n = slot_bytes(desc, s);
        memcpy(out + off, src->*s.member, n);
        off += n;
    }
    memcpy(out, kMagic, 4);
    put32(out + 4, SBL_CONTAINER_VERSION);
    put32(out + 8, as_u32(desc->out_features));
    put32(out + 12, as_u32(desc->in_features));
    put32(out + 16, as_u32(desc->n));
    put32(out + 20, as_u32(desc->m));
    put32(out + 24, formats);
    uint32_t gb;
    memcpy(&gb, &gamma, 4);
    put32(out + 28, gb);
    put64(out + 32, total - SBL_CONTAINER_HEADER_BYTES);
    put32(out + 48, as_u32(sbl_version()));
    put64(out + kHashAt, image_hash(out, total));  // last: it covers every other byte
    return SBL_OK;
}

sbl_status sbl_container_info(const void *src, size_t src_bytes, sbl_layer_desc *desc, uint32_t *formats,
                              float *gamma)
{
    return parse(src, src_bytes, desc, formats, gamma);
}

sbl_status sbl_container_read(const void *src, size_t src_bytes, const sbl_host_buffers *dst)
{
    if (!dst) return SBL_ERR_INVALID_ARG;
    sbl_layer_desc d;
    uint32_t f = 0;
    const sbl_status st = parse(src, src_bytes, &d, &f, nullptr);
    if (st != SBL_OK) return st;
    for (const Slot &s : kSlots)
        if ((f & s.format) && !(dst->*s.member)) return SBL_ERR_INVALID_ARG;
    const uint8_t *in = static_cast<const uint8_t *>(src);
    size_t off = SBL_CONTAINER_HEADER_BYTES;
    for (const Slot &s : kSlots) {
        if (!(f & s.format)) continue;
        off = round_up(off, kAlign);
        const size_t n = slot_bytes(&d, s);
        memcpy(dst->*s.member, in + off, n);
        off += n;
    }
    return SBL_OK;
}

}  // extern "C"

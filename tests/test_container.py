"""The packed-layer container (include/sbl.h): host code only, so it runs
here without a GPU.  The layout is checked field by field against its
documentation (with an independent FNV-1a and offset computation), the
buffers round-trip bit for bit (the oracle's packed formats of a seeded
layer), and every kind of damage is refused before anything is copied."""
import struct

import numpy as np
import pytest
import torch

import oracle
from sparsity_sbl_quantize_b200 import workloads as wl


@pytest.fixture(scope="module")
def sbl():
    from sparsity_sbl_quantize_b200 import build
    build.build()
    from sparsity_sbl_quantize_b200 import sbl as mod
    return mod


ORDER = ["pk2", "nm_values", "nm_bitmap", "i8", "bf16t", "sp24_values", "sp24_meta", "t24_lo", "t24_hi"]


def fnv1a64(data: bytes) -> int:
    h = 0xcbf29ce484222325
    for b in data:
        h = ((h ^ b) * 0x100000001b3) & 0xFFFFFFFFFFFFFFFF
    return h


def oracle_packed(sbl, O, K, n, m, seed=3):
    """A Packed of CPU tensors holding the oracle's formats of a seeded layer."""
    layer = oracle.Layer(wl.master_weights(O, K, seed=seed), n, m)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a))  # noqa: E731
    vals, bm = oracle.pack_nm(layer.weff, layer.mask, n, m)
    bf16t = (layer.weff.T.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)  # exact for {-1, 0, 1}
    p = sbl.Packed(gamma=torch.tensor([layer.gamma, 0, 0, 0], dtype=torch.float32),
                   pk2=t(oracle.pack_pk2(layer.weff)), nm_values=t(vals), nm_bitmap=t(bm), i8=t(layer.weff),
                   bf16t=t(bf16t.view(np.int16)).view(torch.bfloat16))
    fm = sbl.SBL_FMT_PK2 | sbl.SBL_FMT_NM | sbl.SBL_FMT_I8 | sbl.SBL_FMT_BF16T
    if n <= 2:
        sv, sm = oracle.pack_sp24(layer.weff, layer.mask)
        lo, hi = oracle.pack_t24(layer.weff)
        p.sp24_values, p.sp24_meta, p.t24_lo, p.t24_hi = t(sv), t(sm), t(lo), t(hi)
        fm |= sbl.SBL_FMT_SP24 | sbl.SBL_FMT_T24
    return layer, p, fm


@pytest.mark.parametrize("O,K,n,m", [(48, 96, 2, 4), (528, 1040, 6, 8), (16, 16, 1, 4)])
def test_round_trip_is_bit_exact(sbl, O, K, n, m):
    layer, p, fm = oracle_packed(sbl, O, K, n, m)
    d = sbl.desc(O, K, n, m)
    image = sbl.sbl_container_write(d, fm, layer.gamma, p)
    assert len(image) == sbl.sbl_container_bytes(d, fm)
    d2, f2, g2 = sbl.sbl_container_info(image)
    assert (d2.out_features, d2.in_features, d2.n, d2.m) == (O, K, n, m) and f2 == fm
    assert np.float32(g2).view(np.uint32) == np.float32(layer.gamma).view(np.uint32)
    dst = sbl.alloc_packed(d, fm, device="cpu")
    for name in ORDER:
        if getattr(dst, name) is not None:
            getattr(dst, name).zero_()
    sbl.sbl_container_read(image, dst)
    for name in ORDER:
        a, b = getattr(p, name), getattr(dst, name)
        assert (a is None) == (b is None), name
        if a is not None:
            assert torch.equal(a.view(torch.uint8), b.view(torch.uint8)), name


def test_layout_matches_its_documentation(sbl):
    """Header fields at their documented offsets, little-endian; buffers in
    the documented order, each at a multiple of 64 bytes, zeros between; the
    hash is 64-bit FNV-1a of every byte except its own eight."""
    O, K, n, m = 48, 96, 2, 4
    layer, p, fm = oracle_packed(sbl, O, K, n, m)
    d = sbl.desc(O, K, n, m)
    image = sbl.sbl_container_write(d, fm, layer.gamma, p)
    assert image[:4] == b"SBLP"
    version, o, k, nn, mm, fmt, gbits, payload, h, lib = struct.unpack_from("<IiiiiIIQQi", image, 4)
    assert (version, o, k, nn, mm, fmt) == (1, O, K, n, m, fm)
    assert gbits == int(np.float32(layer.gamma).view(np.uint32))
    assert payload == len(image) - 64 and h == fnv1a64(image[:40] + image[48:])
    assert lib == sbl.sbl_version() and image[52:64] == bytes(12)
    off = 64
    for name in ORDER:
        t = getattr(p, name)
        start = (off + 63) // 64 * 64
        assert start == off, f"{name}: every buffer is a multiple of 256 bytes, so none needs fill"
        raw = t.contiguous().view(torch.uint8).numpy().tobytes()
        assert image[start:start + len(raw)] == raw, name
        off = start + len(raw)
    assert off == len(image)


def test_damage_is_refused(sbl):
    O, K, n, m = 48, 96, 2, 4
    layer, p, fm = oracle_packed(sbl, O, K, n, m)
    d = sbl.desc(O, K, n, m)
    image = bytearray(sbl.sbl_container_write(d, fm, layer.gamma, p))

    def status(img):
        try:
            sbl.sbl_container_info(bytes(img))
            return 0
        except sbl.SblError as e:
            return e.status

    assert status(image) == 0
    for pos in (64, 64 + 300, len(image) - 1):          # payload bytes
        bad = bytearray(image)
        bad[pos] ^= 0x01
        assert status(bad) == 1, pos
    for off in (28, 48, 60):                             # gamma, writer version, reserved
        bad = bytearray(image)
        bad[off] ^= 0x01
        assert status(bad) == 1, off
    bad = bytearray(image)
    bad[0:4] = b"SBLQ"
    assert status(bad) == 1                              # magic
    bad = bytearray(image)
    struct.pack_into("<I", bad, 4, 2)
    assert status(bad) == 4                              # a later container version
    bad = bytearray(image)
    struct.pack_into("<i", bad, 12, 100)
    assert status(bad) == 2                              # in_features not a multiple of 16
    bad = bytearray(image)
    struct.pack_into("<I", bad, 24, fm & ~sbl.SBL_FMT_I8)
    assert status(bad) == 1                              # formats that do not match the payload
    assert status(image[:-1]) == 1                       # truncated
    assert status(image[:63]) == 1                       # shorter than the header
    # reading checks first and copies nothing from a damaged image
    dst = sbl.alloc_packed(d, fm, device="cpu")
    dst.pk2.fill_(0xEE)
    bad = bytearray(image)
    bad[-1] ^= 0x80
    with pytest.raises(sbl.SblError):
        sbl.sbl_container_read(bytes(bad), dst)
    assert bool((dst.pk2 == 0xEE).all())


def test_write_argument_checks(sbl):
    O, K = 48, 96
    layer, p, fm = oracle_packed(sbl, O, K, 2, 4)
    d = sbl.desc(O, K, 2, 4)
    with pytest.raises(sbl.SblError) as e:
        sbl.sbl_container_write(d, fm | (1 << 7), layer.gamma, p)
    assert e.value.status == 1                           # unknown format bit
    with pytest.raises(sbl.SblError) as e:
        sbl.sbl_container_write(d, fm, float("nan"), p)
    assert e.value.status == 1                           # non-finite gamma
    p_missing = sbl.Packed(gamma=p.gamma, pk2=None, i8=p.i8)
    with pytest.raises(sbl.SblError) as e:
        sbl.sbl_container_write(d, sbl.SBL_FMT_PK2 | sbl.SBL_FMT_I8, layer.gamma, p_missing)
    assert e.value.status == 1                           # a present format without its buffer
    d68 = sbl.desc(O, K, 6, 8)
    assert sbl.sbl_container_bytes(d68, sbl.SBL_FMT_SP24) == 0
    with pytest.raises(sbl.SblError) as e:
        sbl.sbl_container_write(d68, sbl.SBL_FMT_T24, layer.gamma, p)
    assert e.value.status == 4                           # T24 needs at most two kept per four
    bad = sbl.desc(O, 100, 2, 4)
    assert sbl.sbl_container_bytes(bad, sbl.SBL_FMT_I8) == 0
    with pytest.raises(sbl.SblError) as e:
        sbl.sbl_container_write(bad, sbl.SBL_FMT_I8, layer.gamma, p)
    assert e.value.status == 2
    with pytest.raises(ValueError):
        sbl.sbl_container_write(d, sbl.SBL_FMT_I8, layer.gamma, sbl.Packed(gamma=p.gamma, i8=p.i8.t()))


def test_save_and_load_through_a_file(sbl, tmp_path):
    layer, p, fm = oracle_packed(sbl, 64, 2560, 2, 4)
    d = sbl.desc(64, 2560, 2, 4)
    path = str(tmp_path / "layer.sblp")
    sbl.save_packed(path, d, fm, p)
    d2, f2, p2 = sbl.load_packed(path, device="cpu")
    assert (d2.out_features, d2.in_features, d2.n, d2.m, f2) == (64, 2560, 2, 4, fm)
    assert float(p2.gamma[0]) == layer.gamma
    for name in ORDER:
        assert torch.equal(getattr(p, name).view(torch.uint8), getattr(p2, name).view(torch.uint8)), name


def test_reader_survives_random_damage(sbl):
    """Seeded fuzzing of the reader: random byte flips, truncations and
    header fields (including huge or negative sizes) must each give a status,
    never a crash or a read outside the image; an intact image still reads."""
    import random
    layer, p, fm = oracle_packed(sbl, 32, 64, 2, 4)
    d = sbl.desc(32, 64, 2, 4)
    image = sbl.sbl_container_write(d, fm, layer.gamma, p)
    rnd = random.Random(11)
    dst = sbl.alloc_packed(d, fm, device="cpu")
    outcomes = {}
    for i in range(3000):
        bad = bytearray(image)
        kind = i % 4
        if kind == 0:                                    # flip a few random bytes
            for _ in range(rnd.randint(1, 4)):
                bad[rnd.randrange(len(bad))] ^= rnd.randint(1, 255)
        elif kind == 1:                                  # truncate anywhere
            bad = bad[:rnd.randrange(len(bad))]
        elif kind == 2:                                  # rewrite one header field
            off = rnd.choice([4, 8, 12, 16, 20, 24, 28, 32, 40, 48])
            width = 8 if off in (32, 40) else 4
            bad[off:off + width] = rnd.getrandbits(8 * width).to_bytes(width, "little")
        else:                                            # a plausible but different descriptor
            struct.pack_into("<iiii", bad, 8, rnd.choice([16, 65536, 1 << 20, -16]),
                             rnd.choice([16, 64, 65536, -64]), rnd.randint(-1, 9), rnd.choice([4, 8, 0]))
        try:
            sbl.sbl_container_info(bytes(bad))
            sbl.sbl_container_read(bytes(bad), dst)
            st = 0
        except sbl.SblError as e:
            st = e.status
        outcomes[st] = outcomes.get(st, 0) + 1
    assert set(outcomes) <= {0, 1, 2, 4}
    assert outcomes.get(0, 0) <= 1                       # no damaged image is accepted
    sbl.sbl_container_read(image, dst)
    assert torch.equal(dst.pk2, p.pk2)


def test_every_format_subset_round_trips_random_bytes(sbl):
    """Any valid descriptor and any subset of the formats it allows: random
    buffer bytes come back unchanged, and the image size is the header plus
    the buffers."""
    import random
    rnd = random.Random(7)
    bits = [sbl.SBL_FMT_PK2, sbl.SBL_FMT_NM, sbl.SBL_FMT_I8, sbl.SBL_FMT_BF16T, sbl.SBL_FMT_SP24, sbl.SBL_FMT_T24]
    for trial in range(60):
        m = rnd.choice([4, 8])
        n = rnd.randint(1, m)
        O = 16 * rnd.randint(1, 12)
        K = 16 * rnd.randint(1, 20)
        if K % m:
            continue
        d = sbl.desc(O, K, n, m)
        allowed = [b for b in bits if n <= 2 or b not in (sbl.SBL_FMT_SP24, sbl.SBL_FMT_T24)]
        fm = 0
        for b in allowed:
            if rnd.random() < 0.5:
                fm |= b
        src = sbl.alloc_packed(d, fm, device="cpu")
        total = 64
        for name in ORDER:
            t = getattr(src, name)
            if t is not None:
                t.view(torch.uint8).copy_(torch.randint(0, 256, t.view(torch.uint8).shape, dtype=torch.uint8))
                total += t.numel() * t.element_size()
        g = rnd.uniform(-1.0, 1.0)
        image = sbl.sbl_container_write(d, fm, g, src)
        assert len(image) == total == sbl.sbl_container_bytes(d, fm)
        d2, f2, g2 = sbl.sbl_container_info(image)
        assert (d2.out_features, d2.in_features, d2.n, d2.m, f2) == (O, K, n, m, fm)
        assert g2 == float(np.float32(g))
        dst = sbl.alloc_packed(d, fm, device="cpu")
        sbl.sbl_container_read(image, dst)
        for name in ORDER:
            a, b = getattr(src, name), getattr(dst, name)
            if a is not None:
                assert torch.equal(a.view(torch.uint8), b.view(torch.uint8)), (trial, name)

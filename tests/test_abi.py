"""C-ABI checks that need no GPU: the library loads, exports every symbol the
header declares, validates arguments on the host and sizes storage exactly."""
import os
import re

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L(librq_built):
    return librq_built


def _header_functions():
    src = open(os.path.join(ROOT, "include", "librq.h")).read()
    return sorted(set(re.findall(r"\b(rq_[a-z0-9_]+)\s*\(", src)))


def test_exports_every_declared_symbol(L):
    lib = L.load()
    names = _header_functions()
    assert len(names) >= 16
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(L.SYMBOLS)
    assert L.rq_abi_version() == 3


def test_status_strings(L):
    for s in range(7):
        assert L.rq_status_string(s).startswith("RQ_")


def _lay(L, **kw):
    base = dict(num_layers=1, num_loops=4, batch=8, kv_heads=16, head_dim=128, max_tokens=4096,
                bits=(2, 2, 2, 4), group=(32, 32, 32, 32))
    base.update(kw)
    return L.make_layout(**base)


def test_layout_validation(L):
    assert L.rq_layout_validate(_lay(L)) == L.RQ_OK
    bad = [dict(num_loops=0), dict(num_loops=33), dict(batch=0), dict(head_dim=48),
           dict(bits=(3, 2, 2, 4)), dict(group=(8, 32, 32, 32)), dict(group=(32, 32, 32, 256)),
           dict(max_tokens=0), dict(num_layers=0)]
    for kw in bad:
        assert L.rq_layout_validate(_lay(L, **kw)) == L.RQ_ERR_INVALID_ARG, kw
    assert L.rq_layout_validate(_lay(L, head_dim=256)) == L.RQ_ERR_UNSUPPORTED
    assert L.rq_layout_validate(_lay(L, head_dim=32)) == L.RQ_ERR_UNSUPPORTED
    lay = _lay(L)
    lay.policy = 7
    assert L.rq_layout_validate(lay) == L.RQ_ERR_INVALID_ARG
    for pol in (L.RQ_POLICY_LAST_LOOP, L.RQ_POLICY_NEXT_LOOP, L.RQ_POLICY_FIRST_LOOP,
                L.RQ_POLICY_PREVIOUS_LOOP):
        assert L.rq_layout_validate(_lay(L, policy=pol)) == L.RQ_OK
        assert L.rq_layout_validate(_lay(L, policy=pol, flags=L.RQ_FLAG_UNIT_ALPHA)) == L.RQ_OK
        assert L.rq_layout_validate(_lay(L, policy=pol, flags=L.RQ_FLAG_META16)) == L.RQ_OK
    assert L.rq_layout_validate(_lay(L, flags=4)) == L.RQ_ERR_INVALID_ARG
    assert L.rq_cache_bytes(_lay(L, batch=0)) == 0


def test_anchor_position_follows_the_policy(L):
    """The anchor component (no LS coefficient, laid out first) is loop L-1
    under Last-/Next-loop and loop 0 under First-/Previous-loop; the layer
    size is the same (bits mirrored)."""
    bits, group = (2, 2, 2, 4), (32, 16, 32, 64)
    last = L.rq_cache_bind(_lay(L, bits=bits, group=group), 1 << 20, 1 << 30)
    first = L.rq_cache_bind(_lay(L, bits=bits[::-1], group=group[::-1],
                                 policy=L.RQ_POLICY_FIRST_LOOP), 1 << 20, 1 << 30)
    assert last.layer_bytes == first.layer_bytes
    assert last.comp_off[3] == 0 and first.comp_off[0] == 0
    rec = lambda c, r: c.rec_bytes[r]
    for r in range(4):
        assert rec(last, r) == rec(first, 3 - r)
    # the anchor record carries no alpha: 32 tokens x (codes + meta) only
    assert rec(first, 0) == 32 * (128 * 4 // 8 + (128 // 64) * 4)
    assert rec(first, 1) == 32 * (128 * 2 // 8 + (128 // 32) * 4 + 2)
    # with the loops ascending after the anchor
    assert first.comp_off[1] < first.comp_off[2] < first.comp_off[3]


@pytest.mark.parametrize("bits,group", [((2, 2, 2, 4), (32,) * 4), ((4, 2, 2, 4), (32,) * 4),
                                        ((2,) * 7 + (4,), (64,) * 8), ((2, 2, 2, 4), (16, 16, 16, 32))])
def test_cache_bytes_equal_effective_bits(L, bits, group):
    """Stored bytes = sum over loops of (b + 32/g + [residual] 16/D) bits per
    element, the oracle's accounting with fp16 scale + fp16 offset (32-bit metadata)."""
    T = 4096
    lay = _lay(L, num_loops=len(bits), bits=bits, group=group, max_tokens=T)
    elems = 8 * 16 * T * 128
    beff = oracle.effective_bits(bits, group, 128, 32, True)
    want = beff * len(bits) * elems / 8
    got = L.rq_layer_bytes(lay)
    assert want <= got <= want + 256 * 3 * len(bits)     # only alignment padding on top
    assert L.rq_cache_bytes(_lay(L, num_layers=3, num_loops=len(bits), bits=bits, group=group,
                                 max_tokens=T)) == 3 * got


def _golden(name):
    vals = {}
    with open(os.path.join(ROOT, "tests", "golden", name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                k, v = (x.strip() for x in line.split("="))
                vals[k] = float(v)
    return vals


@pytest.mark.parametrize("name,bits,group", [
    ("int2_g32", (2, 2, 2, 2), (32,) * 4), ("int2_g16", (2, 2, 2, 2), (16,) * 4),
    ("int24_g32", (2, 2, 2, 4), (32,) * 4), ("int24_g16", (2, 2, 2, 4), (16, 16, 16, 32))])
def test_meta16_cache_bytes_reproduce_the_pages(L, name, bits, group):
    """With RQ_FLAG_META16 the library's own byte count of a layer gives the
    residual b_eff the pages print for Ouro-1.4B (L = 4, D = 128):
    2.6 / 3.1 / 3.1 / 3.5 bits per element [RQ App. A.3, §5.1], and 19.3% of
    BF16 for INT2/4 at g = 32 [RQ-summary]."""
    g = _golden("pages_storage.txt")
    T = 4096
    lay = _lay(L, num_loops=4, bits=bits, group=group, max_tokens=T, flags=L.RQ_FLAG_META16)
    elems = 8 * 16 * T * 128 * 4          # batch 8, 16 heads, T tokens, D 128, 4 loops
    beff = L.rq_layer_bytes(lay) * 8 / elems
    assert beff == pytest.approx(oracle.effective_bits(bits, group, 128, 16, True), abs=1e-3)
    assert round(beff, 1) == g[f"beff_residual_{name}"]
    if name == "int24_g32":
        assert round(beff / 16, 3) == g["storage_frac_int24_residual_g32"]


def test_host_checks_reject_before_launch(L):
    """Invalid arguments return an error status without touching the device."""
    lay = _lay(L, max_tokens=100)
    nb = L.rq_cache_bytes(lay)
    assert L.rq_decode_workspace_bytes(lay, 100) > 0
    with pytest.raises(L.RQError) as e:
        L.rq_cache_bind(lay, 0, 0)
    assert e.value.status == L.RQ_ERR_INVALID_ARG
    with pytest.raises(L.RQError) as e:
        L.rq_cache_bind(lay, 4096 + 8, 8192)          # misaligned base
    assert e.value.status == L.RQ_ERR_INVALID_ARG
    cache = L.rq_cache_bind(lay, 1 << 20, 1 << 30)    # never dereferenced below
    for args, status in [((0, 0, 1 << 12, 90, 20), L.RQ_ERR_CAPACITY),
                         ((0, 0, 1 << 12, -1, 2), L.RQ_ERR_INVALID_ARG),
                         ((1, 0, 1 << 12, 0, 2), L.RQ_ERR_INVALID_ARG),
                         ((0, 2, 1 << 12, 0, 2), L.RQ_ERR_INVALID_ARG),
                         ((0, 0, None, 0, 2), L.RQ_ERR_INVALID_ARG),
                         ((0, 0, (1 << 12) + 2, 0, 2), L.RQ_ERR_INVALID_ARG)]:
        with pytest.raises(L.RQError) as e:
            L.rq_quantize_anchor(cache, *args, stream=0)
        assert e.value.status == status, args
    with pytest.raises(L.RQError) as e:
        L.rq_quantize_append_residual(cache, 0, 0, 3, 1 << 12, 0, 2, stream=0)   # 3 is the anchor
    assert e.value.status == L.RQ_ERR_INVALID_ARG
    for args, status in [((0, None, None, 0, 2), L.RQ_ERR_INVALID_ARG),      # no side
                         ((0, 1 << 12, None, 90, 20), L.RQ_ERR_CAPACITY),
                         ((1, 1 << 12, 1 << 13, 0, 2), L.RQ_ERR_INVALID_ARG),  # layer
                         ((0, None, (1 << 12) + 8, 0, 2), L.RQ_ERR_INVALID_ARG),
                         ((0, 1 << 12, None, -3, 2), L.RQ_ERR_INVALID_ARG)]:
        with pytest.raises(L.RQError) as e:
            L.rq_quantize_append_loops(cache, *args, stream=0)
        assert e.value.status == status, args
    with pytest.raises(L.RQError) as e:
        L.rq_decode_attention(cache, 0, 0, 256, 256, 101, 256, 256, 0.0, 256, 256, 1 << 30,
                              stream=0)
    assert e.value.status == L.RQ_ERR_CAPACITY
    with pytest.raises(L.RQError) as e:
        L.rq_decode_attention(cache, 0, 0, 256, 256, 100, 256, 256, 0.0, 256, 256, 16, stream=0)
    assert e.value.status == L.RQ_ERR_WORKSPACE
    with pytest.raises(L.RQError) as e:
        L.rq_decode_attention(cache, 0, 4, 256, 256, 100, 256, 256, 0.0, 256, 256, 1 << 30,
                              stream=0)
    assert e.value.status == L.RQ_ERR_INVALID_ARG
    with pytest.raises(L.RQError) as e:
        L.rq_decode_attention_bf16(1, 1, 96, 256, 256, 256, 10, 256, 10, 256, 256, 0.0, 256, 256,
                                   1 << 20, stream=0)
    assert e.value.status == L.RQ_ERR_UNSUPPORTED
    for args in [(256, 1 << 20, 0), (256, 1 << 20, 1001), (256 + 4, 1 << 20, 5), (0, 1 << 20, 5),
                 (256, 8, 5)]:
        with pytest.raises(L.RQError) as e:
            L.rq_selftest_wait_timeout(*args, stream=0)
        assert e.value.status == L.RQ_ERR_INVALID_ARG, args


def test_rotation_setter_checks(L):
    """rq_cache_set_rotations: NULL keeps the Hadamard transform, pointers must
    be 16-byte aligned, and head_dim must be 128 (host checks, no launch)."""
    lay = L.make_layout(2, 4, 2, 3, 128, 100, (2, 2, 2, 4), (32,) * 4)
    cache = L.rq_cache_bind(lay, 1 << 20, 1 << 30)
    assert cache.k_rot is None and cache.v_rot is None
    L.rq_cache_set_rotations(cache, 1 << 16, None)
    assert cache.k_rot == 1 << 16 and cache.v_rot is None
    L.rq_cache_set_rotations(cache, None, None)
    assert cache.k_rot is None
    with pytest.raises(L.RQError) as e:
        L.rq_cache_set_rotations(cache, (1 << 16) + 8, None)
    assert e.value.status == L.RQ_ERR_INVALID_ARG
    lay64 = L.make_layout(1, 4, 1, 2, 64, 100, (2, 2, 2, 4), (32,) * 4)
    c64 = L.rq_cache_bind(lay64, 1 << 20, 1 << 30)
    with pytest.raises(L.RQError) as e:
        L.rq_cache_set_rotations(c64, None, 1 << 16)
    assert e.value.status == L.RQ_ERR_UNSUPPORTED


@pytest.mark.parametrize("sms,ctas", [(148, 5), (148, 6), (132, 4), (1, 1)])
def test_split_plan_host_logic(L, sms, ctas):
    """The decode split plan (host logic, no device): at least one split, none
    empty, no more than one per 64-token chunk or the 1024 the counters hold,
    and every resident CTA slot filled once when the sequence allows it."""
    for rows in (1, 3, 16, 128, 256, 1280, 40960):
        for T in (0, 1, 63, 64, 65, 777, 4096, 16384, 65536, 1 << 20):
            s, cps = L.rq_plan_splits(rows, T, ctas, sms)
            chunks = (T + 63) // 64
            assert 1 <= s <= max(1, min(chunks, 1024)), (rows, T, s)
            if chunks:
                assert -(-chunks // cps) == s, (rows, T, s, cps)     # no empty split
                assert s * cps >= chunks and (s - 1) * cps < chunks
                want = min(-(-(sms * ctas) // rows), chunks, 1024)
                assert s >= want, (rows, T, s, want)
            else:
                assert (s, cps) == (1, 0)


def test_split_plan_matches_the_measured_launches(L):
    """The plans the benchmark's launches showed on a 148-SM B200 at five
    CTAs per SM: 8 splits for 256 rows and 11 for 128 rows at 16384 tokens."""
    assert L.rq_plan_splits(256, 16384, 5, 148) == (8, 32)
    assert L.rq_plan_splits(128, 16384, 5, 148) == (11, 24)
    for args in [(0, 100, 5, 148), (4, -1, 5, 148), (4, 100, 0, 148), (4, 100, 5, 0)]:
        with pytest.raises(L.RQError) as e:
            L.rq_plan_splits(*args)
        assert e.value.status == L.RQ_ERR_INVALID_ARG


def test_workspace_holds_every_split_plan(L):
    """The decode workspace holds the error word, one counter per (batch, head)
    and the partials (m, l, acc[D]) of the largest split count any device's plan
    can use (one split per 64-token chunk, at most 1024)."""
    for batch, heads, D in ((1, 1, 128), (16, 16, 128), (3, 5, 64), (64, 40, 128)):
        for T in (0, 1, 100, 4096, 16384, 1 << 17):
            lay = L.make_layout(1, 4, batch, heads, D, max(T, 1), (2, 2, 2, 4), (32,) * 4)
            rows = batch * heads
            need = 256 + rows * 4 + rows * max(1, min((T + 63) // 64, 1024)) * (D + 2) * 4
            assert L.rq_decode_workspace_bytes(lay, T) >= need, (batch, heads, D, T)
            for sms, ctas in ((148, 5), (1, 1), (1000, 8)):
                s, _ = L.rq_plan_splits(rows, T, ctas, sms)
                assert 256 + rows * 4 + rows * s * (D + 2) * 4 <= L.rq_decode_workspace_bytes(lay, T)


def test_means_setter_checks(L):
    """rq_cache_set_means: NULL clears, pointers must be 16-byte aligned."""
    cache = L.rq_cache_bind(_lay(L), 1 << 20, 1 << 30)
    L.rq_cache_set_means(cache, 1 << 16, 1 << 17)
    assert cache.k_means == 1 << 16 and cache.v_means == 1 << 17
    L.rq_cache_set_means(cache, None, None)
    assert cache.k_means is None and cache.v_means is None
    with pytest.raises(L.RQError) as e:
        L.rq_cache_set_means(cache, (1 << 16) + 4, None)
    assert e.value.status == L.RQ_ERR_INVALID_ARG


def test_no_cpu_fallback_in_product():
    """The product package never imports the oracle."""
    pkg = os.path.join(ROOT, "residual_bit_kv_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                src = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in src and "from oracle" not in src, f
                assert "rqo_" not in src, f

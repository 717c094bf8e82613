"""Host-side checks of the C ABI library (no GPU): the shared library loads,
exports every function the header declares, its host packer writes the
documented format (pinned by the hand-worked tile and by the oracle's
independent unpacker), and the size / desc-validation functions behave."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import pins_lib
import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = sorted(os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include")) if f.endswith(".h"))


@pytest.fixture(scope="module")
def S():
    import __graft_entry__

    __graft_entry__._load_builder().build()
    import bit_quantized_moe_warp_b200 as S

    return S


def header_functions():
    src = "".join(open(h).read() for h in HEADERS)
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(strata_[a-z0-9_]+)\s*\(", src)))


def test_header_symbols_exported(S):
    names = header_functions()
    assert len(names) >= 18
    lib = ctypes.CDLL(S.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), f"{n} declared in the header but not exported"
    assert sorted(S.EXPORTED) == names, "Python binding and header disagree"


def test_pack_golden_tile(S):
    blob, expects = pins_lib.load_tile_example()
    codes, scales = oracle.unpack_q2_tiled(blob, 64, 64)
    out = np.zeros(1280, np.uint8)
    S.strata_q2_pack(codes, scales, 64, 64, out)
    assert np.array_equal(out, blob), "library packer differs from the hand-worked tile"


def test_pack_golden_q4_tile(S):
    blob, expects = pins_lib.load_tile_example("q4_tile_example.txt", 2304)
    codes, scales = oracle.unpack_q4_tiled(blob, 64, 64)
    out = np.zeros(2304, np.uint8)
    S.strata_q4_pack(codes, scales, 64, 64, out)
    assert np.array_equal(out, blob), "library packer differs from the hand-worked 4-bit tile"


@pytest.mark.parametrize("rows,K", [(64, 64), (128, 64), (256, 128), (64, 768), (384, 256)])
def test_pack_roundtrip_q4_matrix(S, rows, K):
    rng = np.random.default_rng(rows * 11 + K)
    codes = rng.integers(0, 16, (rows, K), dtype=np.uint8)
    scales = (rng.standard_normal((rows, K // 32)) * 0.02).astype(np.float16)
    n = S.strata_q4_matrix_bytes(rows, K)
    assert n == rows * K // 64 * 36
    out = np.zeros(n, np.uint8)
    S.strata_q4_pack(codes, scales, rows, K, out)
    c2, s2 = oracle.unpack_q4_tiled(out, rows, K)
    assert np.array_equal(c2, codes)
    assert np.array_equal(s2.view(np.uint16), scales.view(np.uint16))


@pytest.mark.parametrize("rows,K", [(64, 64), (128, 64), (256, 128), (64, 768), (384, 256)])
def test_pack_roundtrip_matrix(S, rows, K):
    rng = np.random.default_rng(rows * 7 + K)
    codes = rng.integers(0, 4, (rows, K), dtype=np.uint8)
    scales = (rng.standard_normal((rows, K // 32)) * 0.02).astype(np.float16)
    n = S.strata_q2_matrix_bytes(rows, K)
    assert n == rows * K // 64 * 20
    out = np.zeros(n, np.uint8)
    S.strata_q2_pack(codes, scales, rows, K, out)
    c2, s2 = oracle.unpack_q2_tiled(out, rows, K)
    assert np.array_equal(c2, codes)
    assert np.array_equal(s2.view(np.uint16), scales.view(np.uint16))


@pytest.mark.parametrize("bits", [2, 4])
def test_pack_expert_layout(S, bits):
    d, f = 256, 128
    desc = S.make_desc(d, f, 4, 2, 8, bits=bits)
    ex = synth.gen_expert(5, 0, 3, d, f, bits)
    eb = S.strata_moe_expert_bytes(desc)
    assert eb == 3 * d * f // 32 * (10 if bits == 2 else 18)
    out = np.zeros(eb, np.uint8)
    S.strata_moe_pack_expert(desc, ex["gate_codes"], ex["gate_scales"], ex["up_codes"], ex["up_scales"],
                             ex["down_codes"], ex["down_scales"], out)
    got = oracle.unpack_expert(out, d, f, bits)
    assert got["bits"] == ex["bits"] == bits
    for key in ex:
        if key == "bits":
            continue
        a, b = got[key], ex[key]
        if a.dtype == np.float16:
            a, b = a.view(np.uint16), b.view(np.uint16)
        assert np.array_equal(a, b), key


def test_pack_rejects_bad_code(S):
    codes = np.zeros((128, 64), np.uint8)
    codes[3, 5] = 4
    with pytest.raises(S.StrataError) as ei:
        S.strata_q2_pack(codes, np.zeros((128, 2), np.float16), 128, 64, np.zeros(2560, np.uint8))
    assert ei.value.status == S.STRATA_ERR_BAD_BLOB
    S.strata_q4_pack(codes, np.zeros((128, 2), np.float16), 128, 64, np.zeros(4608, np.uint8))  # 4 is a 4-bit code
    codes[3, 5] = 16
    with pytest.raises(S.StrataError) as ei:
        S.strata_q4_pack(codes, np.zeros((128, 2), np.float16), 128, 64, np.zeros(4608, np.uint8))
    assert ei.value.status == S.STRATA_ERR_BAD_BLOB
    d, f = 128, 128
    desc = S.make_desc(d, f, 4, 2, 8, bits=2)
    big = np.full((f, d), 7, np.uint8)
    sc = np.zeros((f, d // 32), np.float16)
    with pytest.raises(S.StrataError) as ei:
        S.strata_moe_pack_expert(desc, big, sc, big, sc, big.T.copy(), sc, np.zeros(3 * d * f // 32 * 10, np.uint8))
    assert ei.value.status == S.STRATA_ERR_BAD_BLOB


def test_desc_validation(S):
    ok = S.make_desc(2048, 768, 512, 10, 8192)
    assert S.strata_moe_expert_bytes(ok) == 1474560
    assert S.strata_moe_expert_blob_bytes(ok) == 1474560 * 512
    assert S.strata_moe_workspace_bytes(ok) > 0
    bad = [S.make_desc(2000, 768, 512, 10, 16), S.make_desc(2048, 700, 512, 10, 16),
           S.make_desc(2048, 768, 0, 1, 16), S.make_desc(2048, 768, 8, 9, 16),
           S.make_desc(2048, 768, 512, 33, 16), S.make_desc(2048, 768, 512, 10, 0),
           S.make_desc(2048, 768, 2048, 10, 16)]
    for dsc in bad:
        assert S.strata_moe_workspace_bytes(dsc) == 0
        assert S.strata_moe_expert_bytes(dsc) == 0
    d2 = S.make_desc(256, 128, 16, 4, 8)
    d2.block_size = 16
    assert S.strata_moe_workspace_bytes(d2) == 0
    d3 = S.make_desc(256, 128, 16, 4, 8)
    d3.weight_format = 3
    assert S.strata_moe_workspace_bytes(d3) == 0
    assert S.strata_q2_matrix_bytes(100, 64) == 0
    assert S.strata_q4_matrix_bytes(64, 100) == 0
    q4 = S.make_desc(2048, 768, 512, 10, 8192, bits=4)
    assert S.strata_moe_expert_bytes(q4) == 2654208
    assert S.strata_moe_workspace_bytes(q4) == S.strata_moe_workspace_bytes(ok)


def test_status_strings(S):
    for code in range(-7, 1):
        assert S.strata_status_string(code)


def test_binding_constants_match_header(S):
    """Every #define the binding restates has the header's value."""
    src = "".join(open(h).read() for h in HEADERS)
    defs = dict(re.findall(r"#define\s+(STRATA_[A-Z0-9_]+)\s+\(?([0-9]+)u?\b", src))
    restated = [n for n in dir(S) if n.startswith("STRATA_") and n in defs]
    assert {"STRATA_Q2_TILE_BYTES", "STRATA_ACCUMULATE", "STRATA_FORCE_PREFILL",
            "STRATA_DECODE_MAX_TOKENS", "STRATA_FMT_Q2_0_TILED", "STRATA_FMT_Q4_0_TILED",
            "STRATA_Q4_TILE_BYTES", "STRATA_KV4_BLOCK"} <= set(restated)
    for n in restated:
        assert getattr(S, n) == int(defs[n]), n


def test_checked_build_exports_the_same_calls(S):
    """The checked build is the same library with bounds checks compiled in:
    it exports every call the header declares and says which build it is."""
    import __graft_entry__

    path = __graft_entry__._load_builder().build(checked=True)
    lib = ctypes.CDLL(path)
    for n in header_functions():
        assert hasattr(lib, n), f"{n} missing from the checked build"
    lib.strata_is_checked_build.restype = ctypes.c_int32
    assert lib.strata_is_checked_build() == 1
    assert S.strata_is_checked_build() == 0


def test_kv4_sizes_and_refusals(S):
    """Sizes of the 4-bit KV format and the codec's argument checks, all of
    which return before any device work (no GPU needed)."""
    assert S.strata_kv4_code_bytes(1000, 128) == 64000
    assert S.strata_kv4_scale_bytes(1000, 128) == 8000
    assert S.strata_kv4_code_bytes(3, 256) == 384 and S.strata_kv4_scale_bytes(3, 64) == 12
    assert S.strata_kv4_code_bytes(10, 96) == 0 and S.strata_kv4_scale_bytes(-1, 128) == 0
    for D in (32, 96, 512, 0):
        with pytest.raises(S.StrataError) as e:
            S.strata_kv4_encode(0x1000, 4, D, 0x2000, 0x3000, stream=0)
        assert e.value.status == S.STRATA_ERR_UNSUPPORTED
        with pytest.raises(S.StrataError) as e:
            S.strata_kv4_decode(0x2000, 0x3000, 4, D, 0x1000, stream=0)
        assert e.value.status == S.STRATA_ERR_UNSUPPORTED
    bad = [dict(x=0x1000, n=-1, c=0x2000, s=0x3000),  # negative row count
           dict(x=0, n=4, c=0x2000, s=0x3000),  # NULL input
           dict(x=0x1000, n=4, c=0, s=0x3000),
           dict(x=0x1000, n=4, c=0x2000, s=0),
           dict(x=0x1008, n=4, c=0x2000, s=0x3000),  # x not 16-byte aligned
           dict(x=0x1000, n=4, c=0x2002, s=0x3000),  # codes not 4-byte aligned
           dict(x=0x1000, n=4, c=0x2000, s=0x3001)]  # scales not 2-byte aligned
    for a in bad:
        with pytest.raises(S.StrataError) as e:
            S.strata_kv4_encode(a["x"], a["n"], 128, a["c"], a["s"], stream=0)
        assert e.value.status == S.STRATA_ERR_INVALID_ARG, a
        with pytest.raises(S.StrataError) as e:
            S.strata_kv4_decode(a["c"], a["s"], a["n"], 128, a["x"], stream=0)
        assert e.value.status == S.STRATA_ERR_INVALID_ARG, a
    # zero rows: nothing to do, even with NULL buffers
    S.strata_kv4_encode(0, 0, 128, 0, 0, stream=0)
    S.strata_kv4_decode(0, 0, 0, 128, 0, stream=0)

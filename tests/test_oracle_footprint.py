"""Oracle pin: the KV footprint closed form against the KVSplit page's printed table."""
import os

import pytest

from oracle import footprint_bytes, footprint_bytes_layers, used_bytes, kv_bytes_per_token_layer, block_bytes, MIB

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
BITS = {"FP16": (16, 16), "K8V8": (8, 8), "K8V4": (8, 4), "K4V8": (4, 8), "K4V4": (4, 4)}
SHAPE = dict(n_layers=22, n_kv_heads=4, head_dim=64)   # the table's model shape (a reading)


def _rows(name):
    out = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                out.append(line.split())
    return out


@pytest.mark.parametrize("cfg,tokens,mib", [(r[0], int(r[1]), float(r[2]))
                                            for r in _rows("kvsplit_memory_table.txt")])
def test_footprint_matches_printed_table(cfg, tokens, mib):
    kb, vb = BITS[cfg]
    got = footprint_bytes(k_bits=kb, v_bits=vb, n_tokens=tokens, **SHAPE)
    assert round(got / MIB, 2) == mib


def test_table_rows_are_exact_at_8192_and_4096():
    # at whole-page token counts the printed two decimals are exact, not rounded
    for cfg, tokens, mib in _rows("kvsplit_memory_table.txt"):
        tokens = int(tokens)
        if tokens % 256:
            continue
        kb, vb = BITS[cfg]
        assert footprint_bytes(k_bits=kb, v_bits=vb, n_tokens=tokens, **SHAPE) == float(mib) * MIB


def test_block_bytes_closed_form():
    # 34 B per 8-bit block, 18 B per 4-bit block, 2 B per fp16 element
    assert block_bytes(8, 32) == 34 and block_bytes(4, 32) == 18 and block_bytes(16, 32) == 64
    assert kv_bytes_per_token_layer(4, 64, 16, 16) == 1024
    assert kv_bytes_per_token_layer(4, 64, 8, 8) == 544
    assert kv_bytes_per_token_layer(4, 64, 8, 4) == 416
    assert kv_bytes_per_token_layer(4, 64, 4, 4) == 288
    with pytest.raises(ValueError):
        block_bytes(8, 48)
    with pytest.raises(ValueError):
        block_bytes(3, 32)


def test_page_rounding_reading_of_the_128_token_row():
    # unpadded, the 128-token row would be half the printed value
    kb, vb = BITS["FP16"]
    assert used_bytes(k_bits=kb, v_bits=vb, n_tokens=128, **SHAPE) / MIB == 2.75
    assert footprint_bytes(k_bits=kb, v_bits=vb, n_tokens=128, **SHAPE) / MIB == 5.50
    assert footprint_bytes(k_bits=kb, v_bits=vb, n_tokens=128, page_tokens=128, **SHAPE) / MIB == 2.75


def test_printed_reductions():
    rows = _rows("kvsplit_reductions.txt")
    fp16 = footprint_bytes(k_bits=16, v_bits=16, n_tokens=8192, **SHAPE)
    for cfg, val in rows:
        kb, vb = BITS[cfg]
        q = footprint_bytes(k_bits=kb, v_bits=vb, n_tokens=8192, **SHAPE)
        if "." in val:   # context multiplier, printed truncated to one decimal
            assert int(fp16 / q * 10) / 10 == float(val)
        else:
            assert round(100 * (1 - q / fp16)) == int(val)


def _table_mib(cfg, tokens):
    for c, t, mib in _rows("kvsplit_memory_table.txt"):
        if c == cfg and int(t) == tokens:
            return float(mib)
    raise KeyError((cfg, tokens))


@pytest.mark.parametrize("mix", [("K8V4", "K4V4"), ("K8V8", "FP16"), ("K8V4", "K4V8")])
@pytest.mark.parametrize("tokens", [8192, 4096])
def test_per_layer_footprint_is_the_layer_share_of_the_printed_rows(mix, tokens):
    """A 22-layer cache with 11 layers of each format holds half of each printed row (exact at whole
    pages): per-layer precision changes bytes layer by layer and nothing else."""
    try:
        want = (_table_mib(mix[0], tokens) + _table_mib(mix[1], tokens)) / 2
    except KeyError:
        pytest.skip("row not printed at this length")
    bits = [BITS[mix[0]]] * 11 + [BITS[mix[1]]] * 11
    got = footprint_bytes_layers(SHAPE["n_kv_heads"], SHAPE["head_dim"], bits, tokens)
    assert got == want * MIB
    # the order of the layers does not matter
    assert footprint_bytes_layers(SHAPE["n_kv_heads"], SHAPE["head_dim"], bits[::-1], tokens) == got


def test_per_layer_footprint_of_uniform_layers_is_the_uniform_closed_form():
    for cfg, kbvb in BITS.items():
        for tokens in (1, 128, 257, 8192):
            assert footprint_bytes_layers(4, 64, [kbvb] * 22, tokens) == footprint_bytes(k_bits=kbvb[0], v_bits=kbvb[1],
                                                                                         n_tokens=tokens, **SHAPE)

"""The FLOP/byte accounting against the cost table the handbook page prints
("Serving several LoRAs, ControlNet and IP-Adapter", section "LoRA: merged or
alongside": FLUX, 57 layers x 4 projections, d = 3072, 4608 tokens)."""
import os

import numpy as np

from adapter_gemv_sgmv_b200 import accounting as acc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "lora_costs_flux.txt")


def _rows():
    out = []
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        r, pct, mb, ms = line.split()
        out.append((int(r), float(pct), int(mb), int(ms)))
    return out


def test_cost_formulas_reproduce_the_printed_flux_table():
    """The page's table, recomputed from the library's per-layer formulas: FLUX has
    57 layers with a LoRA on each of 4 attention projections (d = 3072, square),
    4608 tokens, bf16 weights and an HBM of 3350 GB/s.  Each table column is one
    ratio or sum of those formulas, so a wrong term in any of them shows here."""
    d, n_proj, n_tok, hbm = 3072, 57 * 4, 4608, 3350e9
    rows = _rows()
    assert [r[0] for r in rows] == [8, 16, 64, 128]
    for rank, pct, mb, ms in rows:
        base = 2 * n_tok * d * d                        # one projection's x W^T
        extra = acc.lora_flops(n_tok, rank, d, d) / base
        size_mib = acc.adapter_elems(rank, d, d) * acc.BF16_BYTES * n_proj / 2 ** 20
        merge_s = acc.merge_bytes(d * d * acc.BF16_BYTES * n_proj) / hbm
        assert f"{extra:.1%}" == f"{pct:.1f}%"
        assert round(size_mib) == mb
        assert round(merge_s * 1e3) == ms
        # the extra fraction is exactly 2r/d
        assert abs(extra - 2 * rank / d) < 1e-15


def test_bgmv_cost_counts_distinct_adapters_once():
    ids = np.array([3, 3, 1, -1, 3], np.int32)
    ranks = np.array([8, 16, 8, 32], np.int32)
    c = acc.bgmv_cost(ids, ranks, 64, 32)
    assert c.flops == 2 * (3 * 32 + 16) * (64 + 32)
    assert c.tokens == 4
    assert c.adapter_bytes == 2 * (32 + 16) * (64 + 32)
    assert c.act_bytes == 4 * (2 * 64 + 4 * 32)


def test_multi_cost_single_pass_over_y():
    c = acc.multi_cost(np.array([0, 4, 10]), np.array([0, 2, 3]), np.array([0, 1, 1]),
                       np.array([8, 16]), 32, 32)
    assert c.tokens == 10
    assert c.flops == 2 * 4 * (8 + 16) * 64 + 2 * 6 * 16 * 64
    assert c.act_bytes == 10 * (2 * 32 + 4 * 32)

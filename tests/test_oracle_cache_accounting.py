"""Pins the oracle's closed-form cache accounting to the sizes the pages print
(tests/golden/cache_tables.json, each entry cited there)."""
import json
import os

import pytest

from oracle import cache_accounting as ca

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "cache_tables.json")))


def test_eyestech_telemetry_table():
    g = GOLD["eyestech_pypi_telemetry"]
    for row in g["rows"]:
        if row["kind"] == "mla":
            per = ca.elements_per_token_layer("mla", d_c=row["d_c"], d_rope=row["d_rope"])
        else:
            per = ca.elements_per_token_layer("mha", n_heads=row["n_heads"], d_head=row["d_head"])
        assert per == row["scalars"], row["arch"]
        for ctx, gb in zip(g["contexts"], row["gb"]):
            if row["kind"] == "mla":
                nbytes = ca.compute_kv_cache_bytes(g["n_layers"], 0, 0, ctx, g["batch"],
                                                   g["bytes_per_elem"], is_mla=True,
                                                   d_latent=row["d_c"], d_rope=row["d_rope"])
            else:
                nbytes = ca.compute_kv_cache_bytes(g["n_layers"], row["n_heads"], row["d_head"],
                                                   ctx, g["batch"], g["bytes_per_elem"])
            assert ca.format_gb(nbytes) == gb + " GB", (row["arch"], ctx)


def test_eyestech_api_example():
    g = GOLD["eyestech_pypi_api"]
    kw = dict(n_layers=g["n_layers"], n_kv_heads=g["n_kv_heads"], d_head=g["d_head"],
              seq_len=g["seq_len"], batch_size=g["batch_size"], bytes_per_elem=g["bytes_per_elem"])
    mla = ca.compute_kv_cache_bytes(**kw, is_mla=True, d_latent=g["d_latent"], d_rope=g["d_rope"])
    mha = ca.compute_kv_cache_bytes(**kw, is_mla=False)
    assert ca.format_gb(mla) == g["mla_gb"] + " GB"
    assert ca.format_gb(mha) == g["mha_gb"] + " GB"
    # 67.5 GiB exactly: 576 * 131072 * 8 * 60 * 2 bytes
    assert mla == 67.5 * ca.GIB


def test_eyestech_reduction_percent():
    g = GOLD["eyestech_pypi_reduction"]
    frac = ca.reduction_fraction(g["base_scalars"], g["mla_scalars"])
    assert f"{100 * frac:.2f}" == g["percent"]


def test_from_scratch_table():
    g = GOLD["from_scratch_table"]
    base = ca.elements_per_token_layer("mha", n_heads=g["n_heads"], d_head=g["d_head"])
    for row in g["rows"]:
        per = ca.elements_per_token_layer(row["kind"], n_heads=g["n_heads"], d_head=g["d_head"],
                                          group=row.get("group", 1), d_c=g["d_c"], d_rope=g["d_rope"])
        assert per == row["elements"], row["variant"]
        assert f"{ca.compression_vs(base, per):.2f}" == row["vs"], row["variant"]
        nbytes = per * g["seq_len"] * g["n_layers"] * g["batch"] * g["bytes_per_elem"]
        assert f"{nbytes / ca.GIB:.2f}" == row["gb"], row["variant"]
    # the price of decoupled RoPE: MLA minus MLA-without-RoPE
    rope = (ca.elements_per_token_layer("mla", d_c=g["d_c"], d_rope=g["d_rope"])
            - ca.elements_per_token_layer("mla_no_rope", d_c=g["d_c"]))
    nbytes = rope * g["seq_len"] * g["n_layers"] * g["batch"] * g["bytes_per_elem"]
    assert f"{nbytes / ca.GIB:.2f}" == g["rope_price_gb"]
    # spec figure: 8.44 GB at 128k, 60 layers, fp16 for the V2 shape
    v2 = ca.compute_kv_cache_bytes(60, 32, 128, 131072, 1, 2, is_mla=True, d_latent=512, d_rope=64)
    assert ca.format_gb(v2) == "8.44 GB" and v2 == 8.4375 * ca.GIB


def test_songhuiming_per_sequence():
    g = GOLD["songhuiming_per_sequence"]
    # that page stores k and v of width d (=7168) for MHA and c (=512) for MLA, no RoPE key
    mha = g["n_layers"] * g["n_tokens"] * 2 * g["d"]
    mla = g["n_layers"] * g["n_tokens"] * ca.elements_per_token_layer("mla_no_rope", d_c=g["d_c"])
    assert mha == g["mha_params"] and mla == g["mla_params"]
    assert f"{mha * 2 / ca.MIB:.0f}" == g["mha_mb"]
    assert f"{mla * 2 / ca.MIB:.1f}" == g["mla_mb"]
    assert round(2 * g["d"] / g["d_c"]) == g["ratio_denominator"]


@pytest.mark.parametrize("arch,kw,expect", [
    ("mha", dict(n_heads=128, d_head=128), 32768),
    ("gqa", dict(n_heads=32, d_head=128, group=4), 2048),
    ("mla", dict(d_c=512, d_rope=64), 576),
])
def test_elements_closed_form(arch, kw, expect):
    # 576 elements per token per layer for MLA versus 2 * n_h * d_h for MHA
    assert ca.elements_per_token_layer(arch, **kw) == expect

"""KV-cache ledger of "DeepSeek-V4 Hybrid Attention: CSA and HCA from Scratch".

Test infrastructure only (see oracle/__init__.py).  Section 1 of that page counts the
BF16 GQA8 baseline as K + V: 2 * (8 * 128) * 2 = 4096 bytes per token per layer;
section 12.1 counts it as n * 8 * 128 * 2 = 2048 n bytes (K or V only) and derives its
12.5% / 0.4% / 6.3% ratios from that figure.  The baseline is therefore a parameter.
The pages' ledger leaves out the indexer-key cache; it is reported separately here.
"""
from __future__ import annotations


def kv_ledger(n=1, c=512, m=4, m_prime=128, n_kv_heads=8, d_h=128, elem_bytes=2,
              kv_factor=1, n_csa_layers=30, n_hca_layers=31, cI=128):
    """Per-layer cache bytes and ratios for a context of n tokens.

    kv_factor=1 reproduces section 12.1 (2048 n bytes for GQA8); kv_factor=2 counts
    K and V as in section 1 (4096 bytes per token).
    """
    gqa = n * n_kv_heads * d_h * elem_bytes * kv_factor
    csa = (n / m) * c * elem_bytes
    hca = (n / m_prime) * c * elem_bytes
    layers = n_csa_layers + n_hca_layers
    mix = (n_csa_layers * csa + n_hca_layers * hca) / (layers * gqa)
    indexer_keys = (n / m) * cI * elem_bytes
    return {
        "gqa_bytes": gqa,
        "csa_bytes": csa,
        "hca_bytes": hca,
        "csa_over_gqa": csa / gqa,
        "hca_over_gqa": hca / gqa,
        "mix_over_gqa": mix,
        "indexer_key_bytes": indexer_keys,
    }


def raw_request_bytes(n=10**6, layers=61, bytes_per_token_layer=4096):
    """Raw GQA8 KV bytes for one request (section 1: n * L * 4096)."""
    return n * layers * bytes_per_token_layer

"""Per-token KV-state byte ledger for MHA, GQA and MLA.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

Follows the KV-representation ledger of the datawhalechina tutorial "ARCH-MLA.
Multihead Latent Attention | MLA 与紧凑 KV 表示", section "Step 4：实现 KV 表示账本":
a config needs six positive integer fields and the query heads must divide evenly
over the KV heads; MHA and GQA cache a K and a V per (KV) head; the simplified MLA
caches the latent plus the position component. The same arithmetic gives the
modeldna primer's cache-size table ("Under the hood"): 16,384 / 2,048 / 576 values
per token per layer at 64 heads x 128, 8 KV heads, latent 512, rope 64.
"""
from __future__ import annotations

FIELDS = ("num_heads", "num_kv_heads", "head_dim", "latent_dim", "rope_dim", "dtype_bytes")
MODES = ("mha", "gqa", "mla")


def validate_attention_state_config(config: dict) -> None:
    absent = [f for f in FIELDS if f not in config]
    if absent:
        raise ValueError(f"missing fields: {absent}")
    for f in FIELDS:
        v = config[f]
        if isinstance(v, bool) or not isinstance(v, int) or v <= 0:
            raise ValueError(f"{f} must be a positive integer, got {v!r}")
    if config["num_heads"] % config["num_kv_heads"] != 0:
        raise ValueError("num_heads must be a multiple of num_kv_heads")


def elements_per_token(mode: str, config: dict) -> int:
    validate_attention_state_config(config)
    if mode == "mha":
        return 2 * config["num_heads"] * config["head_dim"]       # K and V for every head
    if mode == "gqa":
        return 2 * config["num_kv_heads"] * config["head_dim"]    # K and V per shared KV head
    if mode == "mla":
        return config["latent_dim"] + config["rope_dim"]          # latent + shared rope key
    raise ValueError(f"unknown mode: {mode}")


def cache_bytes_per_token(mode: str, config: dict) -> int:
    return elements_per_token(mode, config) * config["dtype_bytes"]


def compare_attention_states(config: dict) -> dict:
    per_mode = {m: cache_bytes_per_token(m, config) for m in MODES}
    base = per_mode["mha"]
    return {
        "bytes_per_token": per_mode,
        "ratio_vs_mha": {m: per_mode[m] / base for m in MODES},
        "most_compact": min(MODES, key=lambda m: per_mode[m]),
    }

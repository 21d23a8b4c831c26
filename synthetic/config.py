"""Committed model configs (JSON) -> plain dicts.

The configs fix every choice the Dory pages leave open (head and MLP shapes,
window, SWA:full period, RoPE bases, softmax scale, SwiGLU gate scale, norm
epsilon, alpha initialisation).  Both the oracle and the GPU harness read the
same file as data.
"""

import json
import os

CONFIG_DIR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "configs")

_REQUIRED = (
    "d_model", "n_q_heads", "n_kv_heads", "head_dim", "d_ff",
    "n_in_blocks", "n_rec_blocks", "n_out_blocks", "window", "full_period",
    "rope_base_swa", "rope_base_full", "softmax_scale", "gate_scale", "norm_eps",
    "alpha_init", "weight_std",
)


def load_config(name_or_path, **overrides):
    """Load `configs/<name>.json` (or an explicit path) and apply overrides."""
    path = name_or_path
    if not os.path.isfile(path):
        path = os.path.join(CONFIG_DIR, f"{name_or_path}.json")
    with open(path) as f:
        cfg = json.load(f)
    cfg.update(overrides)
    missing = [k for k in _REQUIRED if k not in cfg]
    if missing:
        raise ValueError(f"config {path} lacks {missing}")
    if cfg["d_model"] != cfg["n_q_heads"] * cfg["head_dim"]:
        raise ValueError("d_model must equal n_q_heads * head_dim")
    if cfg["n_q_heads"] % cfg["n_kv_heads"]:
        raise ValueError("n_q_heads must be a multiple of n_kv_heads")
    return cfg


def n_blocks(cfg):
    return cfg["n_in_blocks"] + cfg["n_rec_blocks"] + cfg["n_out_blocks"]

"""The workload shapes against the values the NucleusMoE-Image walkthrough prints
(``tests/golden/nucleusmoe_image_defaults.txt``, each with its section). CPU only."""

import math
from pathlib import Path

from diffusion_transformer_moe_b200 import inputs as I

GOLDEN = Path(__file__).resolve().parent / "golden" / "nucleusmoe_image_defaults.txt"


def _defaults():
    vals = {}
    for line in GOLDEN.read_text(encoding="utf-8").splitlines():
        line = line.split("#", 1)[0].strip()
        if line:
            k, v = (s.strip() for s in line.split("="))
            vals[k] = float(v) if "." in v else int(v)
    return vals


def test_printed_values_are_consistent_with_each_other():
    g = _defaults()
    assert g["inner_dim"] == g["num_attention_heads"] * g["attention_head_dim"]
    assert g["pixels_per_patch_side"] == g["vae_scale_factor"] * g["patch_size"]
    assert g["default_sample_size"] * g["vae_scale_factor"] == 1024


def _tokens_per_image(g):
    side = g["default_sample_size"] * g["vae_scale_factor"] // g["pixels_per_patch_side"]
    return side * side


def test_1024px_cfg_workloads_are_a_pair_of_default_images():
    g = _defaults()
    S = _tokens_per_image(g)
    assert S == 4096                        # a 64 x 64 patch grid
    for name in ("1024px_cfg", "model_default_1024px_cfg"):
        assert I.WORKLOADS[name].T == 2 * S  # the conditional and unconditional pass


def test_model_default_workload_is_the_printed_configuration():
    g = _defaults()
    w = I.WORKLOADS["model_default_1024px_cfg"]
    S = _tokens_per_image(g)
    assert (w.d, w.E, w.F) == (g["inner_dim"], g["num_experts"], g["moe_intermediate_dim"])
    assert w.capacity_factor == g["capacity_factor"]
    # section 6.2: capacity = ceil(capacity_factor * S / E) tokens per expert per image
    assert w.segments == 2 and w.T // w.segments == S
    assert w.C == math.ceil(g["capacity_factor"] * S / g["num_experts"]) == 256

"""Workload shapes and schedules against the figures and hyper-parameters the page prints."""
import math

from _golden import keyed
from sparsity_mask_sampling_b200 import configs


def test_llama2_7b_block_count_is_the_pages_1_6_billion():
    """All attention and FFN projections of the 32 LLaMA-2-7B layers at 2:4 give 1.6 billion
    blocks of 4 weights, 6 logits each (about 9.6 billion), as the page states."""
    figs = keyed("paper_figures.txt")
    w = configs.WORKLOADS["llama2_7b_stack_2of4"]
    B = w.total_blocks()
    assert B == 32 * (4 * 4096 * 4096 + 3 * 4096 * 11008) // 4 == 1_619_001_344
    assert round(B / 1e9, 1) == float(figs["llama2_7b_blocks_billion"][0])
    assert w.C == int(figs["logits_per_block_2of4"][0])
    assert math.isclose(round(B / 1e9, 1) * w.C, float(figs["llama2_7b_logits_billion"][0]))
    assert configs.WORKLOADS["llama2_7b_layer_2of4"].total_blocks() == 50_593_792
    assert configs.WORKLOADS["general_4of8"].total_blocks() == 2 * 11008 * 4096 // 8 == 11_272_192
    assert configs.WORKLOADS["gpt3_843m_layer_2of4"].total_blocks() == 7_077_888


def test_schedules_and_hyperparameters_follow_table_7():
    hp = {k: float(v[0]) for k, v in keyed("hyperparams.txt").items()}
    w = configs.WORKLOADS["llama2_7b_layer_2of4"]
    assert (w.tau_at(0), w.tau_at(w.steps - 1)) == (hp["tau_start"], hp["tau_end"])
    assert (w.kappa_at(0), w.kappa_at(w.steps - 1)) == (hp["kappa_start"], hp["kappa_end"])
    assert math.isclose(w.tau_at(w.steps // 2), 4 + (0.05 - 4) * (w.steps // 2) / (w.steps - 1))
    assert w.alpha == hp["alpha"] and w.init_std == hp["init_std"] and w.lam == hp["lambda"]
    assert w.lr == hp["lr_llama"] and configs.WORKLOADS["gpt3_843m_layer_2of4"].lr == hp["lr_gpt3"]
    assert all(x.weight_decay == hp["weight_decay"] for x in configs.WORKLOADS.values())
    assert configs.linear_schedule(1.0, 2.0, 0, 1) == 1.0

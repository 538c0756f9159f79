"""Which Linears are quantized: counts printed on the pages."""
import json
import os
import re

from oracle import scope

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "scope_counts.json")))


def test_fp8_dynamic_selects_252():
    names = scope.language_linear_names()
    sel = scope.fp8_dynamic_selected(names)
    assert len(sel) == GOLD["fp8_dynamic_linears"]["value"]
    layers = sorted({int(n.split(".")[3]) for n in sel})
    assert len(layers) == GOLD["fp8_dynamic_layers"]["value"]
    cross = GOLD["cross_attention_layers"]["value"]
    assert list(scope.CROSS_LAYERS) == cross
    assert not set(layers) & set(cross)
    assert scope.N_LAYERS == GOLD["n_language_layers"]["value"]


def test_nf4_keep_ends_selects_240():
    names = scope.language_linear_names()
    sel = scope.nf4_keep_ends_selected(names)
    assert len(sel) == GOLD["nf4_keep_ends_linears"]["value"]
    assert len({int(n.split(".")[3]) for n in sel}) == GOLD["nf4_keep_ends_layers"]["value"]


def test_workload_shapes_match_the_pages():
    from fp8_w8a8_dynamic_b200 import workloads as W
    assert W.HIDDEN == GOLD["hidden_size"]["value"]
    assert W.N_HEADS == GOLD["n_query_heads"]["value"]
    assert W.N_KV_HEADS == GOLD["n_kv_heads"]["value"]
    assert len(W.SELF_LAYERS) * len(W.LAYER_LINEARS) == GOLD["fp8_dynamic_linears"]["value"]
    assert list(W.CROSS_LAYERS) == GOLD["cross_attention_layers"]["value"]


def test_target_pattern_selects_the_same_252():
    """The recipe's target pattern, applied to every language Linear and to
    names it must not take (vision tower, lm_head, cross-attention modules,
    the extra `model.` level of the SGLang ignore list, suffixes, other
    projections), selects exactly the walked set."""
    names = scope.language_linear_names()
    decoys = ["model.visual.blocks.0.attn.qkv", "model.language_model.lm_head", "lm_head",
              "model.language_model.model.layers.0.self_attn.q_proj",
              "model.language_model.layers.0.self_attn.q_proj.weight",
              "model.language_model.layers.0.self_attn.q_norm",
              "model.language_model.layers.2.self_attn.q_proj",
              "model.language_model.layers.48.mlp.up_proj",
              "model.language_model.layers.10.mlp.gate_proj",
              "xmodel.language_model.layers.0.mlp.down_proj"]
    pat = re.compile(scope.fp8_dynamic_target_pattern())
    by_pattern = [n for n in names + decoys if pat.fullmatch(n)]
    assert by_pattern == scope.fp8_dynamic_selected(names)
    assert len(by_pattern) == GOLD["fp8_dynamic_linears"]["value"]

"""Which language-model Linears the FP8_DYNAMIC scheme quantizes.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Restated from the "MOSS-VL quantization README", FP8-Dynamic recipe section:
the q/k/v/o projections and the gate/up/down MLP projections of every
language-model layer WITHOUT cross-attention are quantized; MOSS-VL-0708 has
48 language layers with cross-attention at 2, 6, ..., 46.  The NF4 Keep-4
section of the same README skips the first 4 and last 4 layers, and every
``cross_attn`` module, instead.

The module-name model (a cross-attention layer keeps an MLP; its attention
lives under ``cross_attn``) is this project's reading of the README's two
module lists; the count 240 of the NF4 section pins it.
"""

N_LAYERS = 48
CROSS_LAYERS = tuple(range(2, N_LAYERS, 4))
ATTN_PROJ = ("q_proj", "k_proj", "v_proj", "o_proj")
MLP_PROJ = ("gate_proj", "up_proj", "down_proj")


def language_linear_names(n_layers: int = N_LAYERS, cross=CROSS_LAYERS):
    names = []
    for i in range(n_layers):
        base = f"model.language_model.layers.{i}"
        attn = "cross_attn" if i in cross else "self_attn"
        names += [f"{base}.{attn}.{p}" for p in ATTN_PROJ]
        names += [f"{base}.mlp.{p}" for p in MLP_PROJ]
    return names


def fp8_dynamic_selected(names, cross=CROSS_LAYERS):
    """Names the FP8_DYNAMIC scheme quantizes, by walking each name."""
    out = []
    for nm in names:
        parts = nm.split(".")
        layer = int(parts[3])
        if layer in cross:
            continue
        if parts[4] == "self_attn" and parts[5] in ATTN_PROJ:
            out.append(nm)
        elif parts[4] == "mlp" and parts[5] in MLP_PROJ:
            out.append(nm)
    return out


def fp8_dynamic_target_pattern(cross=CROSS_LAYERS, n_layers: int = N_LAYERS) -> str:
    """The recipe's target as a regular expression over module names (the
    README's FP8-Dynamic recipe targets one pattern: a language-model layer
    index from the layers without cross-attention, then a self-attention
    q/k/v/o projection or an MLP gate/up/down projection, anchored at both
    ends).  Built here from this module's own tuples; ``re.fullmatch`` with
    it must select exactly what ``fp8_dynamic_selected`` selects."""
    layers = "|".join(str(i) for i in range(n_layers) if i not in cross)
    attn = "|".join(ATTN_PROJ)
    mlp = "|".join(MLP_PROJ)
    return rf"model\.language_model\.layers\.({layers})\.(self_attn\.({attn})|mlp\.({mlp}))"


def nf4_keep_ends_selected(names, keep: int = 4, n_layers: int = N_LAYERS):
    """Names the NF4 Keep-4 recipe quantizes: every language Linear except
    those in the first/last ``keep`` layers and those under ``cross_attn``."""
    out = []
    for nm in names:
        parts = nm.split(".")
        layer = int(parts[3])
        if layer < keep or layer >= n_layers - keep:
            continue
        if parts[4] == "cross_attn":
            continue
        out.append(nm)
    return out

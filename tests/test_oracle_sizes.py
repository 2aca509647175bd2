"""Size formulas pinned to the byte identities printed on the pages."""
import oracle
from conftest import golden_lines


def _golden():
    return {ln.split()[0]: float(ln.split()[1]) for ln in golden_lines("storage_identities.txt")}


# Mamba-2 8B shapes (d_model 4096, d_inner 8192, 8 groups x d_state 128,
# 128 heads, conv width 4, vocab 256000, 56 layers, untied LM head).
D_MODEL, D_INNER, NG, DS, NH, CONV, VOCAB, LAYERS = 4096, 8192, 8, 128, 128, 4, 256000, 56
IN_PROJ_N = 2 * D_INNER + 2 * NG * DS + NH            # 18560
LARGE = [(IN_PROJ_N, D_MODEL), (D_MODEL, D_INNER)] * LAYERS + [(VOCAB, D_MODEL)] * 2
CONV_DIM = D_INNER + 2 * NG * DS
SMALL_PER_LAYER = [CONV_DIM * CONV, CONV_DIM, NH, NH, NH, D_INNER, D_MODEL]  # conv w/b, A_log, D, dt_bias, gated norm, norm
SMALL = SMALL_PER_LAYER * LAYERS + [D_MODEL]          # + final norm


def test_mamba2_8b_counts():
    g = _golden()
    assert IN_PROJ_N == 18560
    assert len(LARGE) == g["large_matrices"] and len(SMALL) == g["small_fp16_tensors"]
    p_large = sum(n * k for n, k in LARGE)
    p_small = sum(SMALL)
    assert p_large + p_small == g["base_parameters"]
    assert 2 * (p_large + p_small) == g["decoded_fp16_bytes"]


def test_fp4g16_e4m3_payload_identity():
    """codes + one E4M3 byte per 16 + 4-byte FP32 global per matrix + fp16
    small tensors reproduce the printed payload exactly; one fp16 scale per
    group would not."""
    g = _golden()
    small_bytes = 2 * sum(SMALL)
    e4 = sum(oracle.data_bytes(oracle.FMT_FP4G16_E4M3, n, k) + oracle.scale_bytes(oracle.FMT_FP4G16_E4M3, n, k)
             for n, k in LARGE) + 4 * len(LARGE) + small_bytes
    assert e4 == g["packed_payload_bytes"]
    f16 = sum(oracle.data_bytes(oracle.FMT_FP4G16_F16, n, k) + oracle.scale_bytes(oracle.FMT_FP4G16_F16, n, k)
              for n, k in LARGE) + small_bytes
    assert f16 != g["packed_payload_bytes"] and f16 == 5153048576
    params = g["base_parameters"]
    assert round(e4 * 8 / params, 3) == g["bits_per_parameter_about"]


def test_iq4nl_sizes():
    g = _golden()
    assert oracle.data_bytes(oracle.FMT_IQ4_NL, 1, 32) == g["iq4nl_block_bytes"]
    assert oracle.scale_bytes(oracle.FMT_IQ4_NL, 1, 32) == 0
    assert 8 * oracle.data_bytes(oracle.FMT_IQ4_NL, 1, 32) / g["iq4nl_block_weights"] == 4.5
    assert oracle.data_bytes(oracle.FMT_IQ4_NL, 256, 512) == 73728
    gu = oracle.data_bytes(oracle.FMT_IQ4_NL, 1792, 2560)
    dn = oracle.data_bytes(oracle.FMT_IQ4_NL, 2560, 896)
    assert (gu, dn) == (2580480, 1290240) and 32 * (gu + dn) == 123863040
    # the IQ4_NL model file is consistent with 4.5 bits per weight plus a
    # small remainder of FP32 tensors and metadata (not an exact identity)
    bits = g["iq4nl_file_bytes"] * 8 / g["iq4nl_file_parameters"]
    assert 4.5 <= bits < 4.51


def test_fp4_sizes():
    assert oracle.data_bytes(oracle.FMT_FP4G16_F16, 18560, 4096) + oracle.scale_bytes(oracle.FMT_FP4G16_F16, 18560, 4096) == 47513600
    assert oracle.data_bytes(oracle.FMT_FP4G16_E4M3, 18560, 4096) + oracle.scale_bytes(oracle.FMT_FP4G16_E4M3, 18560, 4096) + 4 == 42762244


def test_mxfp4_sizes():
    """MXFP4 ("1bit.gg zyphra": E8M0 scale byte and 32 E2M1 codes per group):
    16 code bytes and 1 scale byte per 32 weights, 4.25 bits per weight."""
    assert oracle.data_bytes(oracle.FMT_MXFP4, 1, 32) == 16
    assert oracle.scale_bytes(oracle.FMT_MXFP4, 1, 32) == 1
    n, k = 2560, 896
    total = oracle.data_bytes(oracle.FMT_MXFP4, n, k) + oracle.scale_bytes(oracle.FMT_MXFP4, n, k)
    assert total == n * k * 17 // 32 and 8 * total / (n * k) == 4.25

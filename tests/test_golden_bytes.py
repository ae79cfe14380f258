"""The byte figures printed on the pages, reconstructed from the oracle's entry-size rule.

"Pushing KV Cache Compression to 890 Bytes per Token", sec. VII: main KV in E2M1 with one
1-byte E4M3 scale per 16 channels, indexer K in MXFP4 (one 1-byte E8M0 scale per 32); four
owned main KV sets (3 encoder sets at r = 2, 1 decoder set at r = 1) of a 512-channel latent,
indexer head dimension 128. The oracle's rule covers the E4M3/16 format; the MXFP4 indexer
bytes use the same rule with 32-channel scale blocks.
"""
from conftest import golden


def test_entry_bytes_rule(orc):
    assert orc.entry_bytes(256) == 144  # main K||V row of this library: 128 B codes + 16 B scales
    assert orc.entry_bytes(64) == 36
    assert orc.entry_bytes(512) == 288
    assert orc.entry_bytes(0) == 0 and orc.entry_bytes(100) == 0


def test_890_bytes_per_token(orc):
    g = golden("byte_budget.txt")
    main_vals = (g["encoder_owned_sets"] * g["main_latent_channels"] // g["encoder_ratio"]
                 + g["decoder_owned_sets"] * g["main_latent_channels"] // g["decoder_ratio"])
    idx_vals = (g["encoder_owned_sets"] * g["indexer_head_dim"] // g["encoder_ratio"]
                + g["decoder_owned_sets"] * g["indexer_head_dim"] // g["decoder_ratio"])
    assert main_vals == g["main_kv_values_per_token"]
    main_bytes = orc.entry_bytes(main_vals)
    assert main_bytes == 720
    idx_bytes = idx_vals // 2 + idx_vals // 32  # MXFP4: 4 bits + 1 byte per 32
    assert idx_bytes == 170
    assert main_bytes + idx_bytes == g["global_kv_bytes_per_token"]


def test_counterfactual_and_ratios(orc):
    g = golden("byte_budget.txt")
    per_layer_vals = (g["encoder_csa2_layers"] * (g["main_latent_channels"] + g["indexer_head_dim"]) // g["encoder_ratio"]
                      + g["decoder_csa2_layers"] * (g["main_latent_channels"] + g["indexer_head_dim"]) // g["decoder_ratio"])
    assert per_layer_vals == g["per_layer_fp8_bytes_per_token"]  # FP8: 1 byte per value
    shared_fp8 = g["main_kv_values_per_token"] + 320
    assert round(10 * per_layer_vals / g["global_kv_bytes_per_token"]) == g["total_reduction_x10"]
    assert round(10 * per_layer_vals / shared_fp8) == g["sharing_reduction_x10"]
    assert round(10 * shared_fp8 / g["global_kv_bytes_per_token"]) == g["fp4_reduction_x10"]


def test_v1_anchor_and_pool():
    g = golden("byte_budget.txt")
    assert 2 * g["v1_layers"] * g["v1_kv_heads"] * g["v1_head_dim"] * 2 == g["v1_bytes_per_token"]
    assert g["pool_blocks"] * g["pool_block_positions"] == g["pool_candidates"]

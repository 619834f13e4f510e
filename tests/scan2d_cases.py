"""Small GPU parity cases, chosen to reach every code path (see test_paths_covered)."""

# ---- small shapes covering every path (several strips, ragged tails, chains of blocks) ----
CASES = {
    "tiny": ("tiny", {}),
    "f32_strips_ragged": ("tiny", dict(batch=2, channels=20, N=16, H=37, W=75)),
    "f32_two_blocks": ("tiny", dict(batch=1, channels=9, N=16, H=21, W=200)),
    "f32_long_chain_backpressure": ("tiny", dict(batch=1, channels=8, N=16, H=40, W=1030)),
    "f32_long_chain_backpressure_tma": ("tiny", dict(batch=1, channels=16, N=16, H=40, W=1024)),
    "f32_global_ring_tma": ("tiny", dict(batch=1, channels=16, N=16, H=37, W=1056)),
    "bf16_k1_tma": ("small", dict(batch=2, channels=20, H=9, W=48)),
    "bf16_N4_tma": ("small", dict(batch=1, channels=8, N=4, H=5, W=16)),
    "bf16_14x14": ("small", dict(batch=3, channels=19, H=14, W=14)),
    "bf16_7x33": ("small", dict(batch=2, channels=8, H=7, W=33)),
    "bf16_k4_in_block": ("vision", dict(batch=2, channels=12, H=24, W=40)),
    "bf16_k4_56x56": ("vision", dict(batch=1, channels=16, H=56, W=56)),
    "bf16_k4_across_blocks": ("vision", dict(batch=1, channels=8, H=20, W=300)),
    "bf16_k4_across_blocks_tma": ("vision", dict(batch=1, channels=12, H=18, W=256)),
    "f32_chain_plain": ("tiny", dict(batch=1, channels=9, N=16, H=21, W=199)),
    "f32_k2_across_blocks": ("tiny", dict(batch=1, channels=10, N=8, H=19, W=260, orient_mask=0b1001)),
    "f32_tr_only": ("tiny", dict(batch=1, channels=8, N=16, H=11, W=45, orient_mask=0b0010)),
    "f32_bl_only": ("tiny", dict(batch=1, channels=8, N=16, H=11, W=45, orient_mask=0b0100)),
    "f32_br_only_chain": ("tiny", dict(batch=1, channels=8, N=16, H=9, W=150, orient_mask=0b1000)),
    "f32_tl_br": ("tiny", dict(batch=2, channels=5, N=4, H=13, W=29, orient_mask=0b1001)),
    "H1": ("tiny", dict(batch=1, channels=8, N=16, H=1, W=77)),
    "W1": ("tiny", dict(batch=1, channels=8, N=16, H=77, W=1)),
    "H1W1": ("tiny", dict(batch=2, channels=3, N=5, H=1, W=1)),
    "W16": ("tiny", dict(batch=1, channels=8, N=16, H=10, W=16)),
    "W17": ("tiny", dict(batch=1, channels=8, N=16, H=10, W=17)),
    "W128": ("tiny", dict(batch=1, channels=8, N=16, H=10, W=128)),
    "W129": ("tiny", dict(batch=1, channels=8, N=16, H=10, W=129)),
    "no_dskip": ("tiny", dict(batch=1, channels=8, N=16, H=12, W=40, dskip=False)),
    "random_A": ("giga", dict(channels=8, H=48, W=100, random_A=True)),
    "wsi_mask_recipe": ("wsi", dict(channels=16, H=40, W=56)),
    "giga_recipe_small": ("giga", dict(channels=8, H=64, W=300)),
    # enough channel groups that the planner keeps two channels per lane
    "f32_g2_chain_tma": ("tiny", dict(batch=4, channels=160, N=16, H=6, W=128)),
    "bf16_g2_14x14": ("small", dict(batch=64, channels=80, H=10, W=14)),
    # two chain slots per block, each walking every other orientation
    "bf16_k4_split_plain": ("vision", dict(batch=1, channels=8, H=9, W=44)),
    "bf16_k3_split_plain": ("vision", dict(batch=2, channels=8, H=11, W=41, orient_mask=0b0111)),
    "f32_k2_split_tma": ("tiny", dict(batch=1, channels=8, N=16, H=12, W=48, orient_mask=0b0011)),
    # vertical-then-horizontal scan order
    "f32_vfirst_chain_tma": ("tiny", dict(batch=1, channels=8, N=16, H=13, W=200, vfirst=True)),
    "f32_vfirst_global_ring": ("tiny", dict(batch=1, channels=16, N=16, H=21, W=1056, vfirst=True)),
    "f32_vfirst_plain_flips": ("tiny", dict(batch=1, channels=9, N=16, H=11, W=45, orient_mask=0b1010, vfirst=True)),
    "bf16_vfirst_k4_split": ("vision", dict(batch=1, channels=8, H=20, W=56, vfirst=True)),
    "bf16_vfirst_k4_global": ("vision", dict(batch=1, channels=8, H=14, W=300, vfirst=True)),
}
for n in (1, 3, 5, 8, 12, 17, 32, 33, 64):
    CASES[f"N{n}"] = ("tiny", dict(batch=1, channels=9, N=n, H=9, W=23))
    CASES[f"N{n}_bf16_k4"] = ("vision", dict(batch=1, channels=8, N=n, H=6, W=10))

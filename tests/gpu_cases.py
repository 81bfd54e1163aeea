"""Seeded batches and head shapes shared by the GPU parity tests."""
import mtfm_synth as syn


def edge_batch(seed=1100):
    # zero-token user, no T, no R, no H, exactly one tile, ragged tails, >128 targets
    L = [(0, 0, 1), (1, 0, 0), (0, 3, 0), (5, 0, 4), (128, 0, 0), (100, 28, 1), (129, 1, 3),
         (0, 0, 0), (300, 40, 130), (2, 2, 2)]
    return syn.fixed_batch([a for a, _, _ in L], [b for _, b, _ in L], [c for _, _, c in L], seed)


BATCHES = {
    "tiny": lambda: syn.tiny_batch(1000),
    "pair": lambda: syn.pair_batch(32, 1001),
    "edge": edge_batch,
    "v2_n512": lambda: syn.sweep_batch(512, v2=True, B=6, seed=1003),
    "v1_n2048": lambda: syn.sweep_batch(2048, v2=False, B=2, seed=1003),
    "v2_n1024": lambda: syn.sweep_batch(1024, v2=True, B=3, seed=1004),
}

HEADS = {
    "tiny": syn.TINY_HEADS,                 # Hq 2, Hkv 1, dh 32
    "pair": syn.PAIR_HEADS,                 # Hq 8, Hkv 2, dh 64
    "r1": syn.Heads(2, 2, 64),              # one query head per KV group (tcgen05 kernels at r = 1)
    "r2": syn.Heads(4, 2, 64),              # two query heads per KV group (r = 2)
    "dh128": syn.Heads(4, 1, 128),
    "r8": syn.Heads(8, 1, 32),
    "dh32_r1": syn.Heads(2, 2, 32),         # head_dim 32 on the tcgen05 kernels (64-byte swizzle), r = 1
    "dh32_r4": syn.Heads(4, 1, 32),         # head_dim 32, r = 4
    "r8_dh64": syn.Heads(8, 1, 64),         # r = 8 at head_dim 64: tcgen05 Target kernel, mma.sync Full kernel
    "dh256": syn.Heads(3, 1, 256),          # the 768-wide shape: Hq 3, Hkv 1, dh 256 (forward only)
}

"""Shapes of the GPU parity cases: sizes the oracle finishes in seconds that
still span several tiles and ragged tails, plus the degenerate cases."""
from gqe_inputs import CONFIGS, Dims

# sizes the oracle finishes in seconds; several tiles and ragged tails
SMALL = {
    "tiny_b2_t256": CONFIGS["tiny_b2_t256"],
    "ragged_b3_t300": Dims(B=3, T=300, D=256, G=4, M=2, k=1),
    "pool4_k2_skewed_t384": Dims(B=1, T=384, D=512, G=8, M=4, k=2, bias0=2.0),
    "single_token_b4": Dims(B=4, T=1, D=128, G=2, M=4, k=1),
    "one_group_g1_m8_k2": Dims(B=2, T=200, D=192, G=1, M=8, k=2),
    "k_equals_m_t260": Dims(B=1, T=260, D=128, G=4, M=2, k=2),
    "pool8_k4_t136": Dims(B=2, T=136, D=256, G=8, M=8, k=4),
    # +20 router bias on expert 0: every token picks it, the other experts'
    # segments are empty
    "empty_segments_bias20": Dims(B=2, T=160, D=256, G=4, M=4, k=1, bias0=20.0),
    "one_token_b1_t1": Dims(B=1, T=1, D=128, G=4, M=2, k=1),
}

"""Work counts for S^2-Attn -- TEST INFRASTRUCTURE ONLY (the oracle's FLOP model).

useful_pairs: the (query, key) pairs that grouped causal attention actually
scores -- per group of G tokens, G(G+1)/2 pairs.  This is the O(L^2) -> O(L^2/g)
claim of the "LongLoRA paper notes" page (section 3.3), made exact for the causal
case.  Pinned in tests against brute-force enumeration of an explicit mask.

llama2_7b_attention_share: the attention share of LLaMA2-7B's FLOPs as in the
FLOP breakdown table of the nearauto.com article (ablation section, Table 7:
24.5% at 8192 with full attention, 72.2% at 65536 full, 39.4% at 65536 with
S^2-Attn).  Counting 2 FLOPs per multiply-add: per layer 8 N d^2 for the Q,K,V,O
projections, 6 N d f for the gated FFN, 4 N * (attended keys per query) * d for
QK^T and PV (attended keys = G, non-causal counting), plus 2 N d V for the LM
head.  With d=4096, f=11008, 32 layers, V=32000 and S^2-Attn at G=N/4 this gives
the table's three numbers.
"""


def useful_pairs(B, N, H, G):
    """Causal in-group (query, key) pairs over the whole tensor."""
    assert N % G == 0
    return B * H * (N // G) * G * (G + 1) // 2


def fwd_flops(B, N, H, D, G):
    """Useful forward FLOPs: QK^T and PV, 2 * D FLOPs each per scored pair."""
    return 4 * D * useful_pairs(B, N, H, G)


def bwd_flops(B, N, H, D, G):
    """Useful backward FLOPs: five pair-GEMMs (S recompute, dP, dV, dK, dQ) = 2.5x forward."""
    return 10 * D * useful_pairs(B, N, H, G)


def llama2_7b_attention_share(N, G, d=4096, ffn=11008, layers=32, vocab=32000):
    attn = layers * 4 * N * G * d
    proj = layers * 8 * N * d * d
    mlp = layers * 6 * N * d * ffn
    head = 2 * N * d * vocab
    return attn / (attn + proj + mlp + head)

"""Writes hand_examples.json: closed-form values of single CCA steps on tiny inputs.

Each expected value is the hand derivation stored beside it, evaluated with ``math``
(cos, sin, log, sqrt of the listed numbers).  Nothing here calls the oracle or the CUDA
path, so the fixture pins both from outside.
"""
import json
import math
import os

EX = {
    "_about": "Hand-derived examples of single steps of the CCA layer. Each value follows "
              "from the stated inputs by arithmetic done by hand (cos/sin/log of the listed "
              "angles); none comes from any program in this repository.",
    "seq_conv_taps": {
        "cite": "gist.science explainer of arXiv 2510.04476, 2. Methodology, Core Mechanism, "
                "'Convolutional Mixing' (causal 1-D convolution along the sequence, as in SSMs)",
        "reading": "PyTorch conv1d cross-correlation with k-1 zeros on the left: tap k-1 weighs "
                   "the current token, tap 0 the token k-1 steps back",
        "conv_kernel": 4, "weights": [1, 10, 100, 1000], "p": [1, 2, 3, 4, 5],
        "expected": [1000, 2100, 3210, 4321, 5432],
        "derivation": "a[t] = 1*p[t-3] + 10*p[t-2] + 100*p[t-1] + 1000*p[t]; the digits of a[t] "
                      "list p[t], p[t-1], p[t-2], p[t-3]",
    },
    "qk_mean_group": {
        "cite": "gist.science explainer, 2. Methodology, Core Mechanism, 'Q-K-Mean'; edgentiq, "
                "'How Compressed Convolutional Attention Works' (shares information between "
                "queries and keys)",
        "reading": "q_h += (pq_h + pk_g)/2 with g = h // G (contiguous groups); "
                   "k_g += (mean_{h in g} pq_h + pk_g)/2",
        "n_heads": 4, "n_kv_heads": 2, "pq": [[1, 2, 3, 4]], "pk": [[10, 20]],
        "bq": [[0, 0, 0, 0]], "bk": [[100, 200]],
        "expected_q": [[5.5, 6, 11.5, 12]], "expected_k": [[105.75, 211.75]],
        "derivation": "heads 0,1 pair with kv head 0 (pk = 10), heads 2,3 with kv head 1 "
                      "(pk = 20): q = ((1+10)/2, (2+10)/2, (3+20)/2, (4+20)/2); "
                      "k0 = 100 + ((1+2)/2 + 10)/2 = 105.75, k1 = 200 + ((3+4)/2 + 20)/2 = 211.75",
    },
    "value_shift_rows": {
        "cite": "gist.science explainer, 2. Methodology, Core Mechanism, 'Value-Shift' (values "
                "from the current and the previous token; half of the heads do not see the present)",
        "pv": [[1, 2, 3, 4], [5, 6, 7, 8], [9, 10, 11, 12]],
        "expected": [[1, 2, 0, 0], [5, 6, 3, 4], [9, 10, 7, 8]],
        "derivation": "channels 2,3 (upper half) of row t are channels 2,3 of row t-1, zero for t = 0",
    },
    "rms_norm_3_4": {
        "cite": "gist.science explainer, 'Q-K-Mean' ('when combined with normalization'); read "
                "as RMS normalisation of each latent head vector, eps 1e-6",
        "u": [3, 4], "eps": 1e-6,
        "expected": [3 / math.sqrt(12.5 + 1e-6), 4 / math.sqrt(12.5 + 1e-6)],
        "derivation": "mean(u^2) = (9+16)/2 = 12.5; u / sqrt(12.5 + 1e-6)",
    },
    "rope_d4": {
        "cite": "gist.science explainer, 2. Methodology, 'RoPE Integration' (RoPE applied "
                "directly to the compressed queries and keys); RoFormer rotation, rotate-half "
                "pairing, base 10000",
        "dl": 4, "base": 10000.0, "u": [1, 2, 0, 0], "positions": [0, 1, 2],
        "expected": [
            [1, 2, 0, 0],
            [math.cos(1.0), 2 * math.cos(0.01), math.sin(1.0), 2 * math.sin(0.01)],
            [math.cos(2.0), 2 * math.cos(0.02), math.sin(2.0), 2 * math.sin(0.02)]],
        "derivation": "theta_0 = 10000^0 = 1, theta_1 = 10000^(-2/4) = 0.01; pairs (0,2) and "
                      "(1,3) rotate by t*theta_i: (u0 cos - u2 sin, u1 cos - u3 sin, "
                      "u0 sin + u2 cos, u1 sin + u3 cos)",
    },
    "attention_quarter_three_quarters": {
        "cite": "gist.science/de explainer, 2. Methodik: Softmax(QK^T)V computed in the "
                "compressed space; causal mask; scale 1/sqrt(d~)",
        "dl": 2,
        "q": [[1, 0], [1, 0]],
        "k": [[0, 0], [math.sqrt(2) * math.log(3.0), 0]],
        "v": [[4, 8], [0, -4]],
        "expected": [[4, 8], [1, -1]],
        "derivation": "row 0 sees only key 0: O = v0. Row 1: scores (0, ln 3) after the "
                      "1/sqrt(2) scale, softmax (1/4, 3/4), O = (4,8)/4 + 3(0,-4)/4 = (1, -1)",
    },
}

if __name__ == "__main__":
    out = os.path.join(os.path.dirname(os.path.abspath(__file__)), "hand_examples.json")
    with open(out, "w") as f:
        json.dump(EX, f, indent=1)

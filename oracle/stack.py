"""Per-layer window sizes of the attention stack (oracle side, test infrastructure).

Restates the rule of the "autoresearch" README (gitee), section 5.2.2
"sliding window attention", and of the Russian code review (web3.okx.com),
paragraph on the "SSSL" pattern: the pattern string repeats over layers
(layer l takes character l mod len(pattern)); 'L' is a window of the full
sequence length, 'S' half of it; the last layer is always given the full
window.  Written independently of the product's driver.
"""


def layer_windows(n_layer: int, seq_len: int, pattern: str = "SSSL"):
    pattern = pattern.upper()
    full = seq_len
    half = seq_len // 2
    out = []
    for layer in range(n_layer):
        ch = pattern[layer % len(pattern)]
        if ch == "L":
            out.append(full)
        elif ch == "S":
            out.append(half)
        else:
            raise ValueError("window pattern characters are S or L, got %r" % ch)
    out[-1] = full
    return out

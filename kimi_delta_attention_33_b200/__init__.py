"""KDA forward pass, B200-native (sm_100a).  The binding lives in ``kimi_delta_attention_33_b200.kda``."""

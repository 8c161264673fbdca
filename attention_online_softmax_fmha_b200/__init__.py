"""libattn: B200-native fused attention forward with an online softmax."""

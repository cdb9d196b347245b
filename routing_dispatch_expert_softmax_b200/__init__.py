"""B200-native routed mixture-of-experts layer forward (sm_100a).
"""

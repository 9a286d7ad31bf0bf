"""B200-native hybrid CSA/HCA attention step (DeepSeek-V4), C-ABI CUDA library + binding."""

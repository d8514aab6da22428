"""B200-native paged-KV attention: the C-ABI library libpa.so and its Python binding."""
